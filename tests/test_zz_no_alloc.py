"""hca_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin inside a host program that owns all device
memory, or a serving loop where a device-synchronising cudaMalloc is not
allowed).  Called straight through the C ABI and compared with hca_decode,
the entry point that takes a caller-allocated workspace, on two calls in a
row with different inputs (the second call must not be affected by what the
first left in the shared scratch array).  This file sorts last so that a run
stopping at the first failure has already run every other test."""
import ctypes

import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
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


def test_noalloc_decode_matches_workspace_decode_twice():
    need_gpu()
    lib = hca.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.hca_decode_noalloc.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, ctypes.c_float, vp, vp]
    lib.hca_decode_noalloc.restype = i
    cases = [([131072, 300, 5, 70000, 128 * 40 + 7], 1023, 11),
             ([1, 129, 1000000, 256, 65536, 4000, 131071, 2], 7811, 12)]
    for lens, max_nc, seed in cases:
        q, ck, cv, wk, wv, ctx, g = _case(lens, max_nc, seed)
        got = _noalloc(lib, q, ck, cv, wk, wv, ctx, g)
        ref = hca.decode(q, ck, cv, wk, wv, ctx, g)
        torch.cuda.synchronize()
        assert hca.device_error()[0] == 0
        assert_close_out(to64(got), to64(ref), f"noalloc vs decode lens={lens}")


def test_noalloc_rejects_too_many_sequences():
    need_gpu()
    lib = hca.lib()
    S = 65
    q = torch.zeros((S, 64, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((S, 128, 512), dtype=torch.bfloat16, device="cuda")
    ctx = torch.ones((S,), dtype=torch.int32, device="cuda")
    code = lib.hca_decode_noalloc(q.data_ptr(), None, None, 0, w.data_ptr(), w.data_ptr(),
                                  ctx.data_ptr(), q.data_ptr(), S, 64, ctypes.c_float(0.04),
                                  q.data_ptr(), None)
    assert code == 2  # HCA_ERR_UNSUPPORTED, nothing launched
