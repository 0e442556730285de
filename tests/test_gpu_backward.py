"""hca_prefill_bwd vs the fp64 oracle's backward (every element of every
gradient).

Tolerance, derived from the arithmetic: the kernels hold P, dS and dO in
bf16 (relative rounding 2^-9 each) and accumulate in fp32; the forward's
output and compressed cache they start from are bf16 as well.  dS = P (dP -
D) subtracts two roundings of nearly the same number (dP = bf16(dO) . v,
D = sum dout * out), so its error is about 2^-8 of P |dP| rather than of
|dS|; in a row with n visible keys dP - D keeps sqrt(1 - 1/n) of the spread
of dP, hence a relative error of at most 2^-8 sqrt(2) for n >= 2, plus 2^-8
from the operand roundings: about 1e-2 in the worst case (sequences of two
or three tokens), a few times 2^-9 for long ones.  The bar is relative L2
<= 2e-2 and max-abs <= 2e-2 of the largest magnitude of each gradient.

One exception: a single token sees a single key, its softmax is constant and
the exact dq and dk are 0.  The kernel's dS there is dP - D with
dP = bf16(dO) . v and D = sum dout * out, two roundings of the same number:
|dS| <= 2^-7 |dO| |v| (Cauchy-Schwarz on the 2^-9 relative rounding of dO and
of out), so |dq_d| <= scale 2^-7 |dO| |v| |k_d| and
|dk_d| <= scale 2^-7 |dO| |v| sum_h |q_hd|, which that case checks instead."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import errors, need_gpu, to64

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "ds", "dg")


def _check_device():
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"


def _run(B, T, seed, q_scale=1.0):
    x = I.prefill_inputs(I.PrefillConfig(f"bw{T}", B=B, T=T, seed=seed))
    if q_scale != 1.0:
        x["q"] = (x["q"].float() * q_scale).to(torch.bfloat16)
    dout = I.normal_bf16(seed, "dout", B * T, (64, 512)).reshape(B, T, 64, 512)
    d = {n: t.cuda() for n, t in x.items()}
    ck, cv = hca.compress(d["k"], d["v"], d["s"])
    out, lse = hca.prefill(d["q"], d["k"], d["v"], ck, cv, d["g"], return_lse=True)
    grads = hca.prefill_backward(d["q"], d["k"], d["v"], d["s"], ck, cv, d["g"], out, lse,
                                 dout.cuda())
    _check_device()
    ref = O.prefill_backward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]),
                             to64(x["g"]), to64(dout))
    return x, dout, [to64(t) for t in grads], ref


def _single_key_dq_bound(x, dout, b):
    """Per-element bound on dq at position 0 of sequence b (one key: the exact
    value is 0; see the module docstring)."""
    g = to64(x["g"])[b, 0]
    dO = to64(dout)[b, 0] / (1.0 + np.exp(-g))
    v, k = to64(x["v"])[b, 0], to64(x["k"])[b, 0]
    ds_bound = 2.0 ** -7 * np.linalg.norm(dO, axis=1) * np.linalg.norm(v)
    return ds_bound[:, None] * np.abs(k)[None, :] / np.sqrt(512.0)


def _case(B, T, seed, q_scale=1.0):
    x, dout, grads, ref = _run(B, T, seed, q_scale)
    # position 0 sees one key: its dq is checked against the single-key bound,
    # the other positions against the relative bars
    for b in range(B):
        assert (np.abs(grads[0][b, 0]) <= _single_key_dq_bound(x, dout, b)).all()
    grads[0], ref = grads[0][:, 1:], [ref[0][:, 1:]] + list(ref[1:])
    for name, got, want in zip(NAMES, grads, ref):
        assert np.isfinite(got).all(), f"{name}: non-finite values"
        max_abs, rel = errors(got, want)
        top = float(np.abs(want).max())
        print(f"B={B} T={T} {name}: max_abs={max_abs:.3e} (max {top:.3e}) rel_l2={rel:.3e}")
        assert rel <= 2e-2 and max_abs <= 2e-2 * max(top, 1e-30), \
            f"B={B} T={T} {name}: max_abs={max_abs:.3e} (max {top:.3e}) rel_l2={rel:.3e}"


def test_backward_single_token():
    need_gpu()
    x, dout, (dq, dk, dv, ds, dg), ref = _run(1, 1, seed=9001)
    q, v, g = to64(x["q"])[0, 0], to64(x["v"])[0, 0], to64(x["g"])[0, 0]
    dO = to64(dout)[0, 0] / (1.0 + np.exp(-g))                       # [64, 512]
    scale = 1.0 / np.sqrt(512.0)
    ds_bound = 2.0 ** -7 * np.linalg.norm(dO, axis=1) * np.linalg.norm(v)   # [64]
    assert (np.abs(dq[0, 0]) <= _single_key_dq_bound(x, dout, 0)).all()
    assert (np.abs(dk[0, 0]) <= scale * ds_bound.max() * np.abs(q).sum(0)).all()
    assert not ds.any()                                               # no complete block
    for name, got, want in (("dv", dv, ref[2]), ("dg", dg, ref[4])):
        max_abs, rel = errors(got, want)
        assert rel <= 2e-2 and max_abs <= 2e-2 * np.abs(want).max(), (name, max_abs, rel)


@pytest.mark.parametrize("B,T", [(1, 2), (1, 5), (1, 127), (1, 128), (1, 129), (1, 254),
                                 (1, 255), (1, 256), (2, 300), (1, 640), (1, 1024)])
def test_backward_small_all_elements(B, T):
    need_gpu()
    _case(B, T, seed=9000 + T)


def test_backward_2048_three_key_tiles():
    """T = 2048: 16 compressed entries, several compressed-tile splits."""
    need_gpu()
    _case(1, 2048, seed=9100)


def test_backward_large_scores():
    need_gpu()
    _case(1, 700, seed=9200, q_scale=3.0)
