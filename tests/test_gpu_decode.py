"""hca_decode vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import assert_close_cache, assert_close_out, need_gpu, to64

pytestmark = pytest.mark.gpu


def _direct_case(lens, max_nc, seed):
    cfg = I.DecodeConfig("t", S=len(lens), seed=seed, ctx=1, from_raw=False)
    parts = [I.decode_direct_sequence(cfg, i, max_nc) for i in range(len(lens))]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    return q, g, ck, cv, wk, wv


def _run(q, g, ck, cv, wk, wv, lens):
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = hca.decode(q.cuda(), ck.cuda(), cv.cuda(), wk.cuda(), wv.cuda(), ctx, g.cuda())
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"
    return out


@pytest.mark.parametrize("lens", [[1], [5, 127, 128, 129], [255, 256, 383, 384, 1000],
                                  [128 * 40 + 7, 3, 128 * 17], [20000] * 3 + [1] * 5])
def test_decode_direct_cache(lens):
    need_gpu()
    max_nc = max(1, max(max(0, (L - 128) // 128) for L in lens))
    q, g, ck, cv, wk, wv = _direct_case(lens, max_nc, seed=len(lens) * 31 + lens[0])
    out = _run(q, g, ck, cv, wk, wv, lens)
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, f"lens={lens}")


def test_decode_zero_max_nc():
    """Contexts shorter than 256 need no compressed entry at all."""
    need_gpu()
    lens = [1, 2, 100, 200, 255]
    q, g, _, _, wk, wv = _direct_case(lens, 1, seed=3)
    ck = torch.zeros((len(lens), 0, 512), dtype=torch.bfloat16)
    out = _run(q, g, ck, ck.clone(), wk, wv, lens)
    ref = O.decode_forward(to64(q), np.zeros((len(lens), 0, 512)), np.zeros((len(lens), 0, 512)),
                           to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, "max_nc=0")


def test_decode_long_context_workload():
    """16 sequences, lengths U[65536, 1048576] (seeded), cache drawn directly."""
    need_gpu()
    cfg = I.DECODE_16xLONG
    lens = I.decode_ctx_lens(cfg)
    max_nc = 8191
    parts = [I.decode_direct_sequence(cfg, i, max_nc) for i in range(cfg.S)]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    out = _run(q, g, ck, cv, wk, wv, lens)
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, cfg.name)


def test_decode_cache_from_compress_workload():
    """64 sequences at L = 131072, cache built by hca_compress from raw K/V/s.
    For every sequence the oracle builds its own fp64 cache from the same raw
    inputs; every cache entry and every output row is compared."""
    need_gpu()
    cfg = I.DECODE_64x128K
    L = cfg.ctx
    S = cfg.S
    ck = torch.empty((S, L // 128, 512), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    wk = torch.empty((S, 128, 512), dtype=torch.bfloat16)
    wv = torch.empty_like(wk)
    ref_ck, ref_cv = [], []
    for i in range(S):
        k, v, s = I.decode_raw_sequence(cfg, i, L)
        hca.compress(k[None].cuda(), v[None].cuda(), s[None].cuda(), ck[i:i + 1], cv[i:i + 1])
        wk[i] = I.ring_window(k, L)
        wv[i] = I.ring_window(v, L)
        rck, rcv = O.compress(to64(k)[None], to64(v)[None], to64(s)[None])
        assert_close_cache(to64(ck[i]), rck[0], f"ck seq {i}")
        assert_close_cache(to64(cv[i]), rcv[0], f"cv seq {i}")
        ref_ck.append(rck[0])
        ref_cv.append(rcv[0])
    q, g = I.decode_query(cfg)
    out = _run(q, g, ck, cv, wk, wv, [L] * S)
    ref = O.decode_forward(to64(q), np.stack(ref_ck), np.stack(ref_cv), to64(wk), to64(wv),
                           [L] * S, to64(g))
    assert_close_out(to64(out), ref, cfg.name)
    for i in range(S):
        assert_close_out(to64(out[i:i + 1]), ref[i:i + 1], f"seq {i}")


def test_decode_many_splits_large_scores():
    """Two long sequences spread over every SM (one tile per split), with
    scores that grow along the cache so the splits' running maxima differ by
    many units: bounds the rounding of the bf16 partials and of the f16
    sigmoid in the combine, and exercises the combine's rescaling."""
    need_gpu()
    lens = [1_000_000, 700_001]
    max_nc = (lens[0] - 128) // 128
    q, g, ck, cv, wk, wv = _direct_case(lens, max_nc, seed=77)
    ramp = torch.linspace(0.5, 3.0, max_nc).reshape(1, max_nc, 1)
    ck = (ck.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    out = _run(q, g, ck, cv, wk, wv, lens)
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, "many splits, large scores")


def test_decode_bad_device_length_is_reported_not_faulted():
    need_gpu()
    lens = [300, 10 ** 6]          # the second needs far more entries than max_nc
    q, g, ck, cv, wk, wv = _direct_case(lens, 4, seed=8)
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    hca.decode(q.cuda(), ck.cuda(), cv.cuda(), wk.cuda(), wv.cuda(), ctx, g.cuda())
    code, _ = hca.device_error()
    assert code == 5  # HCA_ERR_DEVICE_INPUT
    assert hca.device_error()[0] == 0  # cleared


@pytest.mark.parametrize("S", [1024, 1025, 1100])
def test_decode_many_sequences_planned_by_plan_kernel(S):
    """Up to 1024 sequences each CTA plans for itself (the prefix in shared
    memory at its largest at S = 1024); above that the tile prefix comes from
    the separate plan kernel."""
    need_gpu()
    rng = np.random.default_rng(11 + S)
    lens = [int(x) for x in rng.integers(1, 700, size=S)]
    max_nc = 4
    q, g, ck, cv, wk, wv = _direct_case(lens, max_nc, seed=12)
    out = _run(q, g, ck, cv, wk, wv, lens)
    ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, f"S={S}")


def test_decode_workspace_reused_across_calls_and_sizes():
    """One zero-filled workspace serves many calls of different S: the grid
    barrier's counter is never reset, so a wrong window would show up as a
    race (different results) on some call."""
    need_gpu()
    ws = hca.decode_workspace(64, torch.device("cuda"))
    cases = []
    for lens, seed in (([3000, 129, 700, 5000, 1], 21), ([20000] * 2 + [300] * 62, 22)):
        max_nc = max(1, max(max(0, (L - 128) // 128) for L in lens))
        args = [t.cuda() for t in _direct_case(lens, max_nc, seed)]
        ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
        cases.append((args, ctx, lens))
    first = []
    for rep in range(12):
        for ci, (args, ctx, lens) in enumerate(cases):
            q, g, ck, cv, wk, wv = args
            out = hca.decode(q, ck, cv, wk, wv, ctx, g, workspace=ws)
            torch.cuda.synchronize()
            if rep == 0:
                first.append(out.clone())
                ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens,
                                       to64(g))
                assert_close_out(to64(out), ref, f"case {ci}")
            else:
                assert torch.equal(out, first[ci]), f"case {ci} rep {rep} differs"
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"
