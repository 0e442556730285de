"""hca_prefill_fwd (after hca_compress) vs the fp64 oracle.

Every output element is compared: small and ragged sequences in one oracle
call, the 32K and 128K workloads (in the launch configuration the benchmark
times) chunk by chunk in a pool of oracle worker processes.
"""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import OUT_MAX_ABS, OUT_REL_L2, assert_close_out, need_gpu, to64
from tests.oracle_pool import prefill_full_errors

pytestmark = pytest.mark.gpu


def _inputs(B, T, seed, k_scale=1.0):
    cfg = I.PrefillConfig(f"t{T}", B=B, T=T, seed=seed, k_scale=k_scale)
    return I.prefill_inputs(cfg)


def _run_gpu(x, return_lse=False):
    d = {n: t.cuda() for n, t in x.items()}
    res = hca.forward(d["q"], d["k"], d["v"], d["s"], d["g"], return_lse=return_lse)
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"
    return res


@pytest.mark.parametrize("B,T", [(1, 1), (1, 2), (1, 3), (1, 17), (1, 127), (1, 128), (1, 129),
                                 (1, 254), (1, 255), (1, 256), (1, 257), (2, 300), (1, 513),
                                 (1, 640)])
def test_prefill_small_all_rows(B, T):
    need_gpu()
    x = _inputs(B, T, seed=7000 + T)
    out = _run_gpu(x)
    ref = O.prefill_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]), to64(x["g"]))
    assert_close_out(to64(out), ref, f"B={B} T={T}")


def test_prefill_tiny_workload_all_rows_and_lse():
    """T = 1024, N(0,1) inputs, seed 0: every row, plus the log-sum-exp."""
    need_gpu()
    x = I.prefill_inputs(I.PREFILL_TINY)
    out, lse = _run_gpu(x, return_lse=True)
    ref, ref_lse = O.prefill_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]),
                                     to64(x["g"]), return_lse=True)
    assert_close_out(to64(out), ref, "T=1024")
    assert np.abs(to64(lse) - ref_lse).max() < 2e-2


def test_prefill_large_scores_need_rescaling():
    """Scores that grow along the sequence force the online-softmax rescale."""
    need_gpu()
    T = 1024
    x = _inputs(1, T, seed=91)
    ramp = torch.linspace(0.2, 3.0, T).reshape(1, T, 1, 1)
    x["q"] = (x["q"].float() * ramp).to(torch.bfloat16)
    out = _run_gpu(x)
    ref = O.prefill_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["s"]), to64(x["g"]))
    assert_close_out(to64(out), ref, "rescale")


def _full_check(cfg):
    x = I.prefill_inputs(cfg)
    out = _run_gpu(x)
    del x
    max_abs, rel, finite = prefill_full_errors(cfg, out)
    print(f"{cfg.name}: every row, max_abs={max_abs:.3e} rel_l2={rel:.3e}")
    assert finite, f"{cfg.name}: non-finite values"
    assert max_abs <= OUT_MAX_ABS and rel <= OUT_REL_L2, \
        f"{cfg.name}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


def test_prefill_32k_all_rows():
    """T = 32768 (K x 0.5): all 32768 x 64 x 512 outputs against the oracle."""
    need_gpu()
    _full_check(I.PREFILL_32K)


def test_prefill_128k_all_rows():
    """T = 131072: all 131072 x 64 x 512 outputs against the oracle."""
    need_gpu()
    _full_check(I.PREFILL_128K)


def test_prefill_last_row_equals_decode():
    """GPU self-consistency: prefill row T-1 == decode at L = T on the same cache."""
    need_gpu()
    T = 1000
    x = _inputs(1, T, seed=4242)
    d = {n: t.cuda() for n, t in x.items()}
    ck, cv = hca.compress(d["k"], d["v"], d["s"])
    out = hca.prefill(d["q"], d["k"], d["v"], ck, cv, d["g"])
    wk = I.ring_window(x["k"][0], T).cuda()[None]
    wv = I.ring_window(x["v"][0], T).cuda()[None]
    dec = hca.decode(d["q"][:, T - 1].contiguous(), ck, cv, wk, wv,
                     torch.tensor([T], dtype=torch.int32, device="cuda"),
                     d["g"][:, T - 1].contiguous())
    torch.cuda.synchronize()
    assert hca.device_error()[0] == 0
    assert_close_out(to64(dec[0]), to64(out[0, T - 1]), "prefill row vs decode")
