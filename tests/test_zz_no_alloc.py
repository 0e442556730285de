"""hca_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin inside a host program that owns all device
memory, or a serving loop where a device-synchronising cudaMalloc is not
allowed).  Called straight through the C ABI, two calls in a row with
different inputs (the second must not be affected by what the first left in
the shared scratch array), each compared with the fp64 oracle and with
hca_decode, the entry point that takes a caller-allocated workspace: both run
the same kernel, so with the same grid (every device with at most
HCA_NOALLOC_MAX_CTAS SMs) the outputs must be bit-identical.  One case uses
the largest S the entry point accepts.  This file sorts last so that a run
stopping at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import assert_close_out, need_gpu, to64

pytestmark = pytest.mark.gpu


def _case(lens, max_nc, seed):
    cfg = I.DecodeConfig("noalloc", S=len(lens), seed=seed, ctx=1, from_raw=False)
    parts = [I.decode_direct_sequence(cfg, i, max_nc) for i in range(len(lens))]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]).cuda() for j in range(4))
    q, g = (t.cuda() for t in I.decode_query(cfg))
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, ck, cv, wk, wv, ctx, g


def _noalloc(lib, q, ck, cv, wk, wv, ctx, g):
    S = q.shape[0]
    out = torch.empty_like(q)
    st = torch.cuda.current_stream().cuda_stream
    code = lib.hca_decode_noalloc(q.data_ptr(), ck.data_ptr(), cv.data_ptr(), ck.shape[1],
                                  wk.data_ptr(), wv.data_ptr(), ctx.data_ptr(), g.data_ptr(),
                                  S, 64, ctypes.c_float(512 ** -0.5), out.data_ptr(), st)
    assert code == 0, hca.STATUS.get(code, code)
    return out


def _bind(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.hca_decode_noalloc.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, ctypes.c_float, vp, vp]
    lib.hca_decode_noalloc.restype = i


def test_noalloc_decode_matches_oracle_and_workspace_decode_twice():
    need_gpu()
    lib = hca.lib()
    _bind(lib)
    same_grid = torch.cuda.get_device_properties(0).multi_processor_count <= 160
    rng = np.random.default_rng(5)
    cases = [([131072, 300, 5, 70000, 128 * 40 + 7], 1023, 11),
             ([1, 129, 1000000, 256, 65536, 4000, 131071, 2], 7811, 12),
             ([int(x) for x in rng.integers(1, 131073, size=64)], 1023, 13)]
    for lens, max_nc, seed in cases:
        q, ck, cv, wk, wv, ctx, g = _case(lens, max_nc, seed)
        got = _noalloc(lib, q, ck, cv, wk, wv, ctx, g)
        torch.cuda.synchronize()
        assert hca.device_error()[0] == 0
        ref = O.decode_forward(to64(q), to64(ck), to64(cv), to64(wk), to64(wv), lens, to64(g))
        assert_close_out(to64(got), ref, f"noalloc vs oracle S={len(lens)}")
        ws_out = hca.decode(q, ck, cv, wk, wv, ctx, g)
        torch.cuda.synchronize()
        assert hca.device_error()[0] == 0
        if same_grid:
            assert torch.equal(got, ws_out), f"noalloc and hca_decode differ, S={len(lens)}"
        else:
            assert_close_out(to64(got), to64(ws_out), f"noalloc vs decode S={len(lens)}")


def test_noalloc_rejects_too_many_sequences():
    need_gpu()
    lib = hca.lib()
    _bind(lib)
    S = 65
    q = torch.zeros((S, 64, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((S, 128, 512), dtype=torch.bfloat16, device="cuda")
    ctx = torch.ones((S,), dtype=torch.int32, device="cuda")
    code = lib.hca_decode_noalloc(q.data_ptr(), None, None, 0, w.data_ptr(), w.data_ptr(),
                                  ctx.data_ptr(), q.data_ptr(), S, 64, ctypes.c_float(0.04),
                                  q.data_ptr(), None)
    assert code == 2  # HCA_ERR_UNSUPPORTED, nothing launched
