"""hca_compress vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import assert_close_cache, need_gpu, to64

pytestmark = pytest.mark.gpu


def _case(B, T, seed, k_scale=1.0, s_scale=1.0):
    k = torch.stack([I.normal_bf16(seed * 10 + b, "k", T, (512,), scale=k_scale) for b in range(B)])
    v = torch.stack([I.normal_bf16(seed * 10 + b, "v", T, (512,)) for b in range(B)])
    s = torch.stack([I.normal_bf16(seed * 10 + b, "s", T, (), scale=s_scale) for b in range(B)])
    return k, v, s


@pytest.mark.parametrize("B,T,s_scale", [(1, 128, 1.0), (1, 1024, 1.0), (2, 300, 1.0),
                                         (3, 1000, 4.0), (1, 4096, 0.0)])
def test_compress_matches_oracle(B, T, s_scale):
    need_gpu()
    k, v, s = _case(B, T, seed=T + B, s_scale=s_scale)
    ck, cv = hca.compress(k.cuda(), v.cuda(), s.cuda())
    torch.cuda.synchronize()
    rk, rv = O.compress(to64(k), to64(v), to64(s))
    assert ck.shape == (B, T // 128, 512)
    assert_close_cache(to64(ck), rk, "ck")
    assert_close_cache(to64(cv), rv, "cv")


def test_compress_no_complete_block_is_noop():
    need_gpu()
    k, v, s = _case(1, 100, seed=5)
    ck, cv = hca.compress(k.cuda(), v.cuda(), s.cuda())
    assert ck.shape == (1, 0, 512)
    assert hca.device_error()[0] == 0


def test_compress_full_32k_cache():
    """The cache of the 32K prefill workload (256 entries, K scaled by 0.5)."""
    need_gpu()
    cfg = I.PREFILL_32K
    base = cfg.seed * 1000
    k = I.normal_bf16(base, "k", cfg.T, (512,), scale=cfg.k_scale)[None]
    v = I.normal_bf16(base, "v", cfg.T, (512,))[None]
    s = I.normal_bf16(base, "s", cfg.T, ())[None]
    ck, cv = hca.compress(k.cuda(), v.cuda(), s.cuda())
    torch.cuda.synchronize()
    rk, rv = O.compress(to64(k), to64(v), to64(s))
    assert_close_cache(to64(ck), rk, "ck")
    assert_close_cache(to64(cv), rv, "cv")
    assert hca.device_error()[0] == 0
