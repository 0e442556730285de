"""FP8 (e4m3) cache: hca_quantize_e4m3 and hca_decode_e4m3 vs the fp64 oracle.

Codes and row scales are integer/rounding decisions taken in fp32 on both
sides, so they must match the oracle bit for bit.  The decode over the
stored cache must match the oracle's decode of the stored values (code times
row scale) within the output tolerance."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import assert_close_out, need_gpu, to64

pytestmark = pytest.mark.gpu


def _quant(x: torch.Tensor):
    codes, scale = hca.quantize_e4m3(x.cuda())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scale.cpu().numpy()


def test_quantizer_codes_and_scales_bit_exact():
    need_gpu()
    rng = np.random.default_rng(3)
    rows = 3000
    x = torch.randn((rows, 512), generator=torch.Generator().manual_seed(5))
    x *= torch.from_numpy(rng.uniform(1e-3, 1e3, (rows, 1)).astype(np.float32))
    x[7] = 0.0                     # an all-zero row: scale 1, codes 0
    x[8] = 0.0
    x[8, 100] = -3.0               # a single nonzero value: coded as -448
    x[9, ::2] = 1e-4               # tiny values next to a large one
    x[9, 1] = 5e4
    xb = x.to(torch.bfloat16)
    codes, scale = _quant(xb)
    ref_codes, ref_scale = O.quantize_e4m3_rows(xb.float().numpy())
    assert np.array_equal(scale, ref_scale)
    assert np.array_equal(codes, ref_codes)
    assert scale[7] == 1.0 and not codes[7].any()
    assert codes[8, 100] == 0xFE                     # -448, the row's largest magnitude
    assert abs(O.e4m3_decode(codes[8, 100]) * scale[8] + 3.0) < 1e-6


def _stored(x: torch.Tensor):
    """GPU codes + scales of bf16 rows and their stored fp64 values."""
    codes, scale = hca.quantize_e4m3(x.cuda())
    return codes, scale, O.dequantize_e4m3_rows(codes.cpu().numpy(), scale.cpu().numpy())


def _run_case(q, g, ck, cv, wk, wv, lens, what):
    c_k, s_k, d_k = _stored(ck)
    c_v, s_v, d_v = _stored(cv)
    w_k, t_k, e_k = _stored(wk)
    w_v, t_v, e_v = _stored(wv)
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = hca.decode_e4m3(q.cuda(), c_k, s_k, c_v, s_v, w_k, t_k, w_v, t_v, ctx, g.cuda())
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"
    ref = O.decode_forward(to64(q), d_k, d_v, e_k, e_v, lens, to64(g))
    assert_close_out(to64(out), ref, what)


def _direct(lens, max_nc, seed, q_scale=1.0):
    cfg = I.DecodeConfig("fp8", S=len(lens), seed=seed, ctx=1, from_raw=False)
    parts = [I.decode_direct_sequence(cfg, i, max_nc) for i in range(len(lens))]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    if q_scale != 1.0:
        q = (q.float() * q_scale).to(torch.bfloat16)
    return q, g, ck, cv, wk, wv


@pytest.mark.parametrize("lens", [[1], [5, 127, 128, 129], [255, 256, 383, 384, 1000],
                                  [128 * 40 + 7, 3, 128 * 17], [20000] * 3 + [1] * 5])
def test_decode_e4m3_direct_cache(lens):
    need_gpu()
    max_nc = max(1, max(max(0, (L - 128) // 128) for L in lens))
    q, g, ck, cv, wk, wv = _direct(lens, max_nc, seed=len(lens) * 13 + lens[0])
    _run_case(q, g, ck, cv, wk, wv, lens, f"lens={lens}")


def test_decode_e4m3_long_context_workload():
    """The 16-sequence long-context workload (lengths U[65536, 1048576]) with
    its cache stored in FP8."""
    need_gpu()
    cfg = I.DECODE_16xLONG
    lens = I.decode_ctx_lens(cfg)
    parts = [I.decode_direct_sequence(cfg, i, 8191) for i in range(cfg.S)]
    ck, cv, wk, wv = (torch.stack([p[j] for p in parts]) for j in range(4))
    q, g = I.decode_query(cfg)
    _run_case(q, g, ck, cv, wk, wv, lens, cfg.name + " fp8")


def test_decode_e4m3_cache_from_compress_workload():
    """64 sequences at L = 131072: cache built by hca_compress, then stored in
    FP8; all 64 outputs against the oracle's decode of the stored values."""
    need_gpu()
    cfg = I.DECODE_64x128K
    L, S = cfg.ctx, cfg.S
    ck = torch.empty((S, L // 128, 512), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    wk = torch.empty((S, 128, 512), dtype=torch.bfloat16)
    wv = torch.empty_like(wk)
    for i in range(S):
        k, v, s = I.decode_raw_sequence(cfg, i, L)
        hca.compress(k[None].cuda(), v[None].cuda(), s[None].cuda(), ck[i:i + 1], cv[i:i + 1])
        wk[i] = I.ring_window(k, L)
        wv[i] = I.ring_window(v, L)
    q, g = I.decode_query(cfg)
    _run_case(q, g, ck.cpu(), cv.cpu(), wk, wv, [L] * S, cfg.name + " fp8")


def test_decode_e4m3_many_splits_large_scores():
    need_gpu()
    lens = [1_000_000, 700_001]
    max_nc = (lens[0] - 128) // 128
    q, g, ck, cv, wk, wv = _direct(lens, max_nc, seed=78, q_scale=2.0)
    ramp = torch.linspace(0.5, 3.0, max_nc).reshape(1, max_nc, 1)
    ck = (ck.float() * ramp).to(torch.bfloat16)
    _run_case(q, g, ck, cv, wk, wv, lens, "fp8 many splits, large scores")


def test_decode_e4m3_zero_max_nc():
    need_gpu()
    lens = [1, 2, 100, 200, 255]
    q, g, _, _, wk, wv = _direct(lens, 1, seed=4)
    empty = torch.zeros((len(lens), 0, 512), dtype=torch.bfloat16)
    _run_case(q, g, empty, empty.clone(), wk, wv, lens, "fp8 max_nc=0")
