"""Host-only checks of the C ABI: the library builds and loads without a GPU,
exports every function include/hca.h declares, and rejects bad arguments
before launching anything (these calls never reach a kernel)."""
import ctypes
import os
import re

import pytest

from compressed_sliding_window_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = B.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(os.path.join(ROOT, "include", "hca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(hca_[a-z0-9_]+)\s*\(", text)
    assert names, "no declarations found"
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_expected_entry_points_declared():
    names = set(declared_functions())
    for n in ("hca_compress", "hca_prefill_fwd", "hca_decode", "hca_decode_workspace_size",
              "hca_get_device_error", "hca_status_string", "hca_version", "hca_cache_append",
              "hca_decode_step", "hca_quantize_e4m3", "hca_decode_e4m3", "hca_prefill_fwd_vha",
              "hca_decode_vha", "hca_prefill_bwd", "hca_prefill_bwd_workspace_size"):
        assert n in names


def test_status_strings(lib):
    lib.hca_status_string.restype = ctypes.c_char_p
    assert lib.hca_status_string(0) == b"HCA_OK"
    assert lib.hca_status_string(1) == b"HCA_ERR_INVALID_ARG"
    assert lib.hca_status_string(4) == b"HCA_ERR_TIMEOUT"
    assert lib.hca_status_string(99) == b"HCA_ERR_UNKNOWN"
    assert lib.hca_version() >= 100


def test_compress_rejects_bad_args(lib):
    lib.hca_compress.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 2 + [ctypes.c_void_p] * 3
    fake = 0x10000
    assert lib.hca_compress(None, fake, fake, 1, 256, fake, fake, None) == 1
    assert lib.hca_compress(fake, fake, fake, 0, 256, fake, fake, None) == 1
    assert lib.hca_compress(fake, fake, fake, 1, 0, fake, fake, None) == 1
    assert lib.hca_compress(fake + 2, fake, fake, 1, 256, fake, fake, None) == 1   # misaligned
    assert lib.hca_compress(fake, fake, fake, 1, 256, None, fake, None) == 1      # no output
    assert lib.hca_compress(fake, fake, fake, 1, 100, None, None, None) == 0      # nb = 0: no-op


def test_prefill_rejects_bad_args(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.hca_prefill_fwd.argtypes = [vp] * 6 + [i, i, i, ctypes.c_float, vp, vp, vp,
                                                ctypes.c_size_t, vp]
    f = 0x10000
    ok_args = [f, f, f, f, f, f, 1, 256, 64, 0.04, f, None, f, 1 << 30, None]

    def call(**kw):
        a = list(ok_args)
        names = ["q", "k", "v", "ck", "cv", "g", "B", "T", "H", "scale", "out", "lse", "ws",
                 "ws_bytes", "st"]
        for k2, v2 in kw.items():
            a[names.index(k2)] = v2
        return lib.hca_prefill_fwd(*a)

    assert call(H=63) == 2
    assert call(B=0) == 1
    assert call(T=0) == 1
    assert call(scale=float("nan")) == 1
    assert call(scale=-1.0) == 1
    assert call(q=None) == 1
    assert call(out=None) == 1
    assert call(ck=None) == 1          # T = 256 has compressed entries
    assert call(g=f + 8) == 1          # misaligned
    assert call(ws=None) == 1          # no workspace
    assert call(ws=f + 16) == 1        # workspace not 256-byte aligned


def test_decode_rejects_bad_args(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.hca_decode.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, ctypes.c_float, vp,
                               ctypes.c_size_t, vp, vp]
    f = 0x10000
    assert lib.hca_decode(f, f, f, 8, f, f, f, f, 4, 32, 0.04, f, 1 << 30, f, None) == 2
    assert lib.hca_decode(f, f, f, 8, f, f, f, f, 0, 64, 0.04, f, 1 << 30, f, None) == 1
    assert lib.hca_decode(None, f, f, 8, f, f, f, f, 4, 64, 0.04, f, 1 << 30, f, None) == 1
    assert lib.hca_decode(f, f, f, 8, f, f, None, f, 4, 64, 0.04, f, 1 << 30, f, None) == 1
    assert lib.hca_decode(f, f, f, -1, f, f, f, f, 4, 64, 0.04, f, 1 << 30, f, None) == 1
    assert lib.hca_decode(f, f, f, 8, f, f, f, f, 4, 64, 0.0, f, 1 << 30, f, None) == 1
    assert lib.hca_decode(f, f, f, 8, f, f, f, f, 4, 64, 0.04, f + 16, 1 << 30, f, None) == 1


def test_cache_append_and_decode_step_reject_bad_arguments(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.hca_cache_append.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, vp, vp, i, vp]
    f = 1 << 20   # aligned fake device address; every call below is rejected on the host
    ok_args = [f, f, f, f, 4, f, f, f, f, f, 8, None]

    def append(**kw):
        a = list(ok_args)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_cache_append(*a)
    assert append(a4=0) == 1                 # S < 1
    assert append(a10=-1) == 1               # max_nc < 0
    assert append(a0=None) == 1              # no k_new
    assert append(a3=None) == 1              # no ctx_len
    assert append(a7=None) == 1              # no score ring
    assert append(a8=None) == 1              # entries needed (max_nc > 0) but no ck
    assert append(a5=f + 8) == 1             # misaligned ring
    lib.hca_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, ctypes.c_float, vp, vp, vp, vp,
                                    vp, i, vp, ctypes.c_size_t, vp, vp]
    base = [f, f, f, f, f, f, 4, 64, 0.04, f, f, f, f, f, 8, f, 1 << 30, f, None]

    def step(**kw):
        a = list(base)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_decode_step(*a)
    assert step(a7=32) == 2                  # H != 64
    assert step(a8=0.0) == 1                 # scale
    assert step(a0=None) == 1                # no q
    assert step(a15=f + 16) == 1             # workspace not 256-byte aligned
    assert step(a2=None) == 1                # no k_new (append half)
    assert step(a6=70000) == 2               # S beyond what decode supports


def test_fp8_entry_points_reject_bad_arguments(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    f = 1 << 20
    lib.hca_quantize_e4m3.argtypes = [vp, ctypes.c_longlong, vp, vp, vp]
    assert lib.hca_quantize_e4m3(f, -1, f, f, None) == 1          # rows < 0
    assert lib.hca_quantize_e4m3(None, 4, f, f, None) == 1        # no input
    assert lib.hca_quantize_e4m3(f + 8, 4, f, f, None) == 1       # misaligned input
    assert lib.hca_quantize_e4m3(f, 4, f, f + 2, None) == 1       # misaligned scales
    assert lib.hca_quantize_e4m3(None, 0, None, None, None) == 0  # nothing to do
    lib.hca_decode_e4m3.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, i, i,
                                    ctypes.c_float, vp, ctypes.c_size_t, vp, vp]
    base = [f, f, f, f, f, 8, f, f, f, f, f, f, 4, 64, 0.04, f, 1 << 30, f, None]

    def call(**kw):
        a = list(base)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_decode_e4m3(*a)
    assert call(a13=32) == 2                 # H != 64
    assert call(a12=0) == 1                  # S < 1
    assert call(a2=None) == 1                # max_nc > 0 but no ck scale
    assert call(a7=None) == 1                # no wk scale
    assert call(a6=f + 4) == 1               # misaligned window codes
    assert call(a14=float("nan")) == 1       # scale


def test_vha_entry_points_reject_bad_arguments(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    f = 1 << 20
    lib.hca_prefill_fwd_vha.argtypes = [vp] * 6 + [i, i, i, ctypes.c_float, vp, vp, i, vp, vp,
                                                    vp, ctypes.c_size_t, vp]
    pre = [f, f, f, f, f, f, 1, 256, 64, 0.04, f, f, 8, f, None, f, 1 << 30, None]

    def prefill(**kw):
        a = list(pre)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_prefill_fwd_vha(*a)
    assert prefill(a12=0) == 1               # rank < 1
    assert prefill(a12=65) == 1              # rank > 64
    assert prefill(a10=None) == 1            # no down factor
    assert prefill(a11=None) == 1            # no up factor
    assert prefill(a8=32) == 2               # H != 64
    assert prefill(a0=None) == 1             # no q
    lib.hca_decode_vha.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, ctypes.c_float, vp, vp,
                                   i, vp, ctypes.c_size_t, vp, vp]
    dec = [f, f, f, 8, f, f, f, f, 4, 64, 0.04, f, f, 4, f, 1 << 30, f, None]

    def decode(**kw):
        a = list(dec)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_decode_vha(*a)
    assert decode(a13=0) == 1                # rank < 1
    assert decode(a13=100) == 1              # rank > 64
    assert decode(a11=None) == 1             # no down factor
    assert decode(a12=None) == 1             # no up factor
    assert decode(a9=32) == 2                # H != 64
    assert decode(a14=f + 16) == 1           # workspace not 256-byte aligned


def test_backward_rejects_bad_arguments(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    f = 1 << 20
    lib.hca_prefill_bwd.argtypes = [vp] * 10 + [i, i, i, ctypes.c_float] + [vp] * 6 + \
        [ctypes.c_size_t, vp]
    base = [f] * 10 + [1, 300, 64, 0.04] + [f] * 6 + [1 << 40, None]

    def call(**kw):
        a = list(base)
        for idx, val in kw.items():
            a[int(idx[1:])] = val
        return lib.hca_prefill_bwd(*a)
    assert call(a12=32) == 2                 # H != 64
    assert call(a10=0) == 1                  # B < 1
    assert call(a11=0) == 1                  # T < 1
    assert call(a13=float("inf")) == 1       # scale
    assert call(a0=None) == 1                # no q
    assert call(a8=None) == 1                # no lse
    assert call(a4=None) == 1                # T = 300 has entries but no ck
    assert call(a14=f + 4) == 1              # misaligned dq
    assert call(a19=f + 16) == 1             # workspace not 256-byte aligned
    assert call(a20=1024) == 1               # workspace too small
    lib.hca_prefill_bwd_workspace_size.argtypes = [i, i]
    lib.hca_prefill_bwd_workspace_size.restype = ctypes.c_size_t
    assert lib.hca_prefill_bwd_workspace_size(0, 10) == 0
    small = lib.hca_prefill_bwd_workspace_size(1, 128)
    big = lib.hca_prefill_bwd_workspace_size(1, 256)
    assert 0 < small < big


def test_selftest_rejects_bad_limit(lib):
    lib.hca_selftest_bounded_wait.argtypes = [ctypes.c_int, ctypes.c_void_p]
    assert lib.hca_selftest_bounded_wait(0, None) == 1
    assert lib.hca_selftest_bounded_wait(10 ** 8, None) == 1


def test_python_binding_fails_loudly_without_gpu():
    import torch
    import compressed_sliding_window_b200 as hca
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    x = torch.zeros((1, 256, 512), dtype=torch.bfloat16)
    s = torch.zeros((1, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hca.compress(x, x, s)


def test_python_binding_checks_new_entry_points_without_gpu():
    """The head-mix and backward bindings refuse host tensors (no CPU
    fallback) and malformed factors before touching the library."""
    import torch
    import compressed_sliding_window_b200 as hca
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    T = 4
    q = torch.zeros((1, T, 64, 512), dtype=torch.bfloat16)
    k = torch.zeros((1, T, 512), dtype=torch.bfloat16)
    s = torch.zeros((1, T), dtype=torch.bfloat16)
    c = torch.zeros((1, 0, 512), dtype=torch.bfloat16)
    lse = torch.zeros((1, T, 64), dtype=torch.float32)
    f = torch.zeros((64, 8), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hca.prefill(q, k, k, c, c, q, vha=(f, f))
    with pytest.raises(ValueError):
        hca.prefill_backward(q, k, k, s, c, c, q, q, lse, q)
    with pytest.raises(ValueError):
        hca.decode(q[0], c, c, torch.zeros((T, 128, 512), dtype=torch.bfloat16),
                   torch.zeros((T, 128, 512), dtype=torch.bfloat16),
                   torch.ones((T,), dtype=torch.int32), q[0], vha=(f, f))
