"""Virtual head attention fused into prefill (hca_prefill_fwd_vha) and decode
(hca_decode_vha) vs the fp64 oracle, which applies the cross-head mix to the
gated output of every position.  Every output element is compared.

Tolerances.  A light mix (factors N(0, 1/16^2): the mixed-in term is at most
a quarter of the gated output at rank 64) keeps the outputs at the size of
the plain attention output, and the plain bar applies (max-abs 2e-2,
relative L2 5e-3).  The kernels mix the gated output as staged in bf16, so
beside the final bf16 rounding of y each element carries one bf16 rounding
of x (|x| 2^-9 at most) and the rounding of the mixing matrix (2^-9 of each
entry): the error bound grows with the output's size.  A strong mix (as large
as the identity or larger) is therefore held to bars relative to the
output's largest magnitude: max-abs <= 1e-2 max|y| (2.5 times the 2^-8 max|y|
that the two roundings reach together) and relative L2 5e-3."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import OUT_REL_L2, assert_close_out, errors, need_gpu, to64

LIGHT = 1.0 / 16

pytestmark = pytest.mark.gpu


def _check_device():
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"


def _assert_close_scaled(got, ref, what):
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_abs, rel = errors(got, ref)
    top = float(np.abs(ref).max())
    assert max_abs <= 1e-2 * top and rel <= OUT_REL_L2, \
        f"{what}: max_abs={max_abs:.3e} (max|y| {top:.3e}) rel_l2={rel:.3e}"


def _prefill_case(B, T, rank, seed, scale=LIGHT, positions=None, strong=False):
    cfg = I.PrefillConfig(f"vha{T}", B=B, T=T, seed=seed)
    x = I.prefill_inputs(cfg)
    down, up = I.vha_factors(rank, seed, scale)
    d = {n: t.cuda() for n, t in x.items()}
    ck, cv = hca.compress(d["k"], d["v"], d["s"])
    out = hca.prefill(d["q"], d["k"], d["v"], ck, cv, d["g"], vha=(down.cuda(), up.cuda()))
    _check_device()
    vha = (to64(down), to64(up))
    if positions is None:
        ref = O.prefill_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]),
                                to64(x["g"]), vha=vha)
        check = _assert_close_scaled if strong else assert_close_out
        check(to64(out), ref, f"B={B} T={T} r={rank}")
    else:
        ref = O.prefill_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]),
                                to64(x["g"]), vha=vha, positions=positions)
        assert_close_out(to64(out[:, positions]), ref, f"B={B} T={T} r={rank} (rows)")


@pytest.mark.parametrize("B,T,rank", [(1, 1, 4), (1, 5, 1), (1, 128, 16), (1, 254, 8),
                                      (2, 300, 64), (1, 1000, 16), (1, 1024, 3)])
def test_prefill_vha_all_rows(B, T, rank):
    need_gpu()
    _prefill_case(B, T, rank, seed=8100 + T + rank)


def test_prefill_vha_strong_mix_4096():
    """A mix as large as the identity (factor scale 1/2, rank 64) over 4096
    positions: every row."""
    need_gpu()
    _prefill_case(1, 4096, 64, seed=8200, scale=0.5, strong=True)


def test_prefill_vha_16k_sampled_rows():
    """T = 16384: rows 0, 1, 126, 127 of every 128-position block and every
    row of the first and last blocks."""
    need_gpu()
    T = 16384
    pos = sorted(set([t for b in range(T // 128) for t in (128 * b, 128 * b + 1, 128 * b + 126,
                                                            128 * b + 127)]
                     + list(range(128)) + list(range(T - 128, T))))
    _prefill_case(1, T, 16, seed=8300, positions=pos)


def test_prefill_vha_matches_plain_kernel_when_mix_is_zero():
    """Zero factors: the fused mix adds exactly zero, so the output equals the
    plain kernel's bit for bit."""
    need_gpu()
    x = I.prefill_inputs(I.PrefillConfig("z", B=1, T=777, seed=8400))
    d = {n: t.cuda() for n, t in x.items()}
    ck, cv = hca.compress(d["k"], d["v"], d["s"])
    plain = hca.prefill(d["q"], d["k"], d["v"], ck, cv, d["g"])
    zero = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    mixed = hca.prefill(d["q"], d["k"], d["v"], ck, cv, d["g"], vha=(zero, zero.clone()))
    _check_device()
    assert torch.equal(plain, mixed)


def _decode_case(lens, rank, seed, scale=LIGHT, strong=False):
    cfg = I.DecodeConfig("vha", S=len(lens), seed=seed, ctx=1, from_raw=False)
    max_nc = max(1, max(max(0, (L - 128) // 128) for L in lens))
    parts = [I.decode_direct_sequence(cfg, i, max_nc) for i in range(len(lens))]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    down, up = I.vha_factors(rank, seed, scale)
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = hca.decode(q.cuda(), ck.cuda(), cv.cuda(), wk.cuda(), wv.cuda(), ctx, g.cuda(),
                     vha=(down.cuda(), up.cuda()))
    _check_device()
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g),
                           vha=(to64(down), to64(up)))
    check = _assert_close_scaled if strong else assert_close_out
    check(to64(out), ref, f"lens={lens[:4]} r={rank}")


@pytest.mark.parametrize("lens,rank", [([1], 4), ([5, 127, 128, 129], 1),
                                       ([255, 256, 383, 384, 1000], 16),
                                       ([128 * 40 + 7, 3, 128 * 17], 64),
                                       ([20000] * 3 + [1] * 5, 8)])
def test_decode_vha(lens, rank):
    need_gpu()
    _decode_case(lens, rank, seed=8500 + rank + len(lens))


def test_decode_vha_strong_mix():
    need_gpu()
    _decode_case([3000, 129, 70000, 1], 64, seed=8550, scale=0.5, strong=True)


def test_decode_vha_many_sequences():
    """300 sequences (more units than CTAs), rank 16."""
    need_gpu()
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 3000, 300)]
    _decode_case(lens, 16, seed=8600)


def test_decode_vha_long_context_workload():
    """The 16-sequence long-context workload (lengths U[65536, 1048576])."""
    need_gpu()
    cfg = I.DECODE_16xLONG
    lens = I.decode_ctx_lens(cfg)
    parts = [I.decode_direct_sequence(cfg, i, 8191) for i in range(cfg.S)]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    down, up = I.vha_factors(16, 4, LIGHT)
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = hca.decode(q.cuda(), ck.cuda(), cv.cuda(), wk.cuda(), wv.cuda(), ctx, g.cuda(),
                     vha=(down.cuda(), up.cuda()))
    _check_device()
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g),
                           vha=(to64(down), to64(up)))
    assert_close_out(to64(out), ref, cfg.name + " vha")


def test_decode_vha_repeatable_on_reused_workspace():
    """Two barriers per launch on one reused workspace: ten launches, one answer."""
    need_gpu()
    lens = [300, 5000, 129, 77777]
    cfg = I.DecodeConfig("vha_rep", S=len(lens), seed=77, ctx=1, from_raw=False)
    parts = [I.decode_direct_sequence(cfg, i, 700) for i in range(len(lens))]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]).cuda() for j in range(4))
    q, g = (t.cuda() for t in I.decode_query(cfg))
    down, up = (t.cuda() for t in I.vha_factors(8, 77))
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = hca.decode_workspace(len(lens), "cuda")
    first = hca.decode(q, ck, cv, wk, wv, ctx, g, workspace=ws, vha=(down, up))
    for _ in range(9):
        again = hca.decode(q, ck, cv, wk, wv, ctx, g, workspace=ws, vha=(down, up))
        assert torch.equal(first, again)
        plain = hca.decode(q, ck, cv, wk, wv, ctx, g, workspace=ws)   # one barrier
    _check_device()
    assert not torch.equal(first, plain)
