"""B200-native Heavily Compressed Attention (HCA) forward path.

Python binding over the C ABI of ``libhca.so`` (declared in include/hca.h).
The functions here only check and marshal arguments (device pointers, sizes,
the current CUDA stream); every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if the library is missing or no CUDA
device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

from .build import LIB_PATH

HEADS = 64
HEAD_DIM = 512
BLOCK = 128
WINDOW = 128

STATUS = {
    0: "HCA_OK", 1: "HCA_ERR_INVALID_ARG", 2: "HCA_ERR_UNSUPPORTED", 3: "HCA_ERR_CUDA",
    4: "HCA_ERR_TIMEOUT", 5: "HCA_ERR_DEVICE_INPUT",
}


class HCAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libhca.so (built in-tree by ``build.py``)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m compressed_sliding_window_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.hca_compress.argtypes = [vp, vp, vp, i, i, vp, vp, vp]
        L.hca_prefill_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, f, vp, vp, vp, sz, vp]
        L.hca_prefill_fwd_vha.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, f, vp, vp, i, vp, vp,
                                          vp, sz, vp]
        L.hca_prefill_workspace_size.argtypes = [i, i]
        L.hca_prefill_workspace_size.restype = sz
        L.hca_decode_workspace_size.argtypes = [i]
        L.hca_decode_workspace_size.restype = sz
        L.hca_decode.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, f, vp, sz, vp, vp]
        L.hca_prefill_bwd_workspace_size.argtypes = [i, i]
        L.hca_prefill_bwd_workspace_size.restype = sz
        L.hca_prefill_bwd.argtypes = [vp] * 10 + [i, i, i, f] + [vp] * 6 + [sz, vp]
        L.hca_decode_vha.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, f, vp, vp, i, vp, sz,
                                     vp, vp]
        L.hca_cache_append.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, vp, vp, i, vp]
        L.hca_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, f, vp, vp, vp, vp, vp, i, vp,
                                      sz, vp, vp]
        L.hca_quantize_e4m3.argtypes = [vp, ctypes.c_longlong, vp, vp, vp]
        L.hca_decode_e4m3.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, i, i, f, vp,
                                      sz, vp, vp]
        L.hca_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
        L.hca_selftest_bounded_wait.argtypes = [i, vp]
        L.hca_status_string.argtypes = [i]
        L.hca_status_string.restype = ctypes.c_char_p
        L.hca_version.restype = i
        for name in ("hca_compress", "hca_prefill_fwd", "hca_decode", "hca_get_device_error",
                     "hca_selftest_bounded_wait", "hca_cache_append", "hca_decode_step",
                     "hca_quantize_e4m3", "hca_decode_e4m3", "hca_prefill_fwd_vha",
                     "hca_decode_vha", "hca_prefill_bwd"):
            getattr(L, name).restype = i
        _LIB = L
    return _LIB


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(t: torch.Tensor, name: str, shape=None, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _ok(fn: str, code: int):
    if code != 0:
        raise HCAError(fn, code)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def compress(k: torch.Tensor, v: torch.Tensor, s: torch.Tensor,
             ck: Optional[torch.Tensor] = None, cv: Optional[torch.Tensor] = None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Compressed cache entries for every complete 128-token block.

    k, v: [B, T, 512] bf16; s: [B, T] bf16 -> (ck, cv) [B, T // 128, 512] bf16.
    """
    B, T, D = k.shape
    _check(k, "k", (B, T, HEAD_DIM))
    _check(v, "v", (B, T, HEAD_DIM))
    _check(s, "s", (B, T))
    nb = T // BLOCK
    if ck is None:
        ck = torch.empty((B, nb, HEAD_DIM), dtype=torch.bfloat16, device=k.device)
    if cv is None:
        cv = torch.empty((B, nb, HEAD_DIM), dtype=torch.bfloat16, device=k.device)
    _check(ck, "ck", (B, nb, HEAD_DIM))
    _check(cv, "cv", (B, nb, HEAD_DIM))
    _ok("hca_compress", lib().hca_compress(k.data_ptr(), v.data_ptr(), s.data_ptr(), B, T,
                                           _ptr(ck) if nb else None, _ptr(cv) if nb else None,
                                           _stream(k.device)))
    return ck, cv


def prefill_workspace_size(B: int, T: int) -> int:
    return int(lib().hca_prefill_workspace_size(B, T))


def _check_vha(vha, device):
    down, up = vha
    r = down.shape[1] if down.dim() == 2 else -1
    _check(down, "vha_down", (HEADS, r))
    _check(up, "vha_up", (HEADS, r))
    if not 1 <= r <= HEADS or down.device != device or up.device != device:
        raise ValueError(f"vha factors must be [64, r] bf16 on {device} with 1 <= r <= 64")
    return down, up, r


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, ck: torch.Tensor,
            cv: torch.Tensor, g: torch.Tensor, scale: Optional[float] = None,
            out: Optional[torch.Tensor] = None, return_lse: bool = False,
            workspace: Optional[torch.Tensor] = None, vha=None):
    """HCA prefill attention with the gate fused.

    q, g: [B, T, 64, 512]; k, v: [B, T, 512]; ck, cv: [B, T // 128, 512]
    -> out [B, T, 64, 512] bf16 (and lse [B, T, 64] fp32 when asked).
    `vha` = (down, up), each [64, r] bf16: virtual head attention fused into
    the epilogue (hca_prefill_fwd_vha).
    """
    B, T, H, D = q.shape
    _check(q, "q", (B, T, H, HEAD_DIM))
    _check(g, "g", (B, T, H, HEAD_DIM))
    _check(k, "k", (B, T, HEAD_DIM))
    _check(v, "v", (B, T, HEAD_DIM))
    nb = T // BLOCK
    _check(ck, "ck", (B, nb, HEAD_DIM))
    _check(cv, "cv", (B, nb, HEAD_DIM))
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (B, T, H, HEAD_DIM))
    lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device) if return_lse else None
    if workspace is None:
        workspace = torch.empty((prefill_workspace_size(B, T),), dtype=torch.uint8,
                                device=q.device)
    _check(workspace, "workspace", dtype=torch.uint8)
    if vha is None:
        _ok("hca_prefill_fwd", lib().hca_prefill_fwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(ck) if nb else None,
            _ptr(cv) if nb else None, g.data_ptr(), B, T, H, ctypes.c_float(scale),
            out.data_ptr(), _ptr(lse), workspace.data_ptr(), workspace.numel(),
            _stream(q.device)))
    else:
        down, up, r = _check_vha(vha, q.device)
        _ok("hca_prefill_fwd_vha", lib().hca_prefill_fwd_vha(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(ck) if nb else None,
            _ptr(cv) if nb else None, g.data_ptr(), B, T, H, ctypes.c_float(scale),
            down.data_ptr(), up.data_ptr(), r, out.data_ptr(), _ptr(lse), workspace.data_ptr(),
            workspace.numel(), _stream(q.device)))
    return (out, lse) if return_lse else out


def prefill_bwd_workspace_size(B: int, T: int) -> int:
    return int(lib().hca_prefill_bwd_workspace_size(B, T))


def prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s: torch.Tensor,
                     ck: torch.Tensor, cv: torch.Tensor, g: torch.Tensor, out: torch.Tensor,
                     lse: torch.Tensor, dout: torch.Tensor, scale: Optional[float] = None,
                     workspace: Optional[torch.Tensor] = None):
    """Gradients of sum(dout * out) for the HCA prefill (hca_prefill_bwd).

    q, g, out, dout: [B, T, 64, 512] bf16; k, v: [B, T, 512]; s: [B, T];
    ck, cv: the forward's compressed cache; lse: [B, T, 64] fp32 from the
    forward.  Returns dq, dg (bf16, shapes of q and g), dk, dv ([B, T, 512]
    fp32) and ds ([B, T] fp32) as (dq, dk, dv, ds, dg).
    """
    B, T, H, D = q.shape
    for t, n in ((q, "q"), (g, "g"), (out, "out"), (dout, "dout")):
        _check(t, n, (B, T, H, HEAD_DIM))
    _check(k, "k", (B, T, HEAD_DIM))
    _check(v, "v", (B, T, HEAD_DIM))
    _check(s, "s", (B, T))
    nb = T // BLOCK
    _check(ck, "ck", (B, nb, HEAD_DIM))
    _check(cv, "cv", (B, nb, HEAD_DIM))
    _check(lse, "lse", (B, T, H), dtype=torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    dq = torch.empty_like(q)
    dg = torch.empty_like(g)
    dk = torch.empty((B, T, HEAD_DIM), dtype=torch.float32, device=q.device)
    dv = torch.empty_like(dk)
    ds = torch.empty((B, T), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty((prefill_bwd_workspace_size(B, T),), dtype=torch.uint8,
                                device=q.device)
    _check(workspace, "workspace", dtype=torch.uint8)
    _ok("hca_prefill_bwd", lib().hca_prefill_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), s.data_ptr(), _ptr(ck) if nb else None,
        _ptr(cv) if nb else None, g.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
        B, T, H, ctypes.c_float(scale), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
        ds.data_ptr(), dg.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream(q.device)))
    return dq, dk, dv, ds, dg


def forward(q, k, v, s, g, scale: Optional[float] = None, return_lse: bool = False):
    """Compress then prefill: the whole HCA forward for a prompt."""
    ck, cv = compress(k, v, s)
    return prefill(q, k, v, ck, cv, g, scale=scale, return_lse=return_lse)


def decode_workspace_size(S: int) -> int:
    return int(lib().hca_decode_workspace_size(S))


def decode_workspace(S: int, device) -> torch.Tensor:
    """A zero-filled decode workspace for up to S sequences (reusable across calls)."""
    return torch.zeros((decode_workspace_size(S),), dtype=torch.uint8, device=device)


def decode(q: torch.Tensor, ck: torch.Tensor, cv: torch.Tensor, wk: torch.Tensor,
           wv: torch.Tensor, ctx_len: torch.Tensor, g: torch.Tensor,
           scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None, vha=None) -> torch.Tensor:
    """One decode step: q, g [S, 64, 512]; ck, cv [S, max_nc, 512]; wk, wv
    [S, 128, 512] ring windows; ctx_len [S] int32 on the device.  A workspace
    passed in comes from ``decode_workspace`` (zero-filled before first use).
    `vha` = (down, up), each [64, r] bf16: virtual head attention fused into
    the same launch (hca_decode_vha)."""
    S, H, D = q.shape
    _check(q, "q", (S, H, HEAD_DIM))
    _check(g, "g", (S, H, HEAD_DIM))
    max_nc = ck.shape[1]
    _check(ck, "ck", (S, max_nc, HEAD_DIM))
    _check(cv, "cv", (S, max_nc, HEAD_DIM))
    _check(wk, "wk", (S, WINDOW, HEAD_DIM))
    _check(wv, "wv", (S, WINDOW, HEAD_DIM))
    _check(ctx_len, "ctx_len", (S,), dtype=torch.int32)
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    if workspace is None:
        workspace = decode_workspace(S, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (S, H, HEAD_DIM))
    _check(workspace, "workspace", dtype=torch.uint8)
    if vha is None:
        _ok("hca_decode", lib().hca_decode(
            q.data_ptr(), _ptr(ck) if max_nc else None, _ptr(cv) if max_nc else None, max_nc,
            wk.data_ptr(), wv.data_ptr(), ctx_len.data_ptr(), g.data_ptr(), S, H,
            ctypes.c_float(scale), workspace.data_ptr(), workspace.numel(), out.data_ptr(),
            _stream(q.device)))
    else:
        down, up, r = _check_vha(vha, q.device)
        _ok("hca_decode_vha", lib().hca_decode_vha(
            q.data_ptr(), _ptr(ck) if max_nc else None, _ptr(cv) if max_nc else None, max_nc,
            wk.data_ptr(), wv.data_ptr(), ctx_len.data_ptr(), g.data_ptr(), S, H,
            ctypes.c_float(scale), down.data_ptr(), up.data_ptr(), r, workspace.data_ptr(),
            workspace.numel(), out.data_ptr(), _stream(q.device)))
    return out


def _check_append(k_new, v_new, s_new, ctx_len, wk, wv, ws, ck, cv):
    S = k_new.shape[0]
    _check(k_new, "k_new", (S, HEAD_DIM))
    _check(v_new, "v_new", (S, HEAD_DIM))
    _check(s_new, "s_new", (S,))
    _check(ctx_len, "ctx_len", (S,), dtype=torch.int32)
    _check(wk, "wk", (S, WINDOW, HEAD_DIM))
    _check(wv, "wv", (S, WINDOW, HEAD_DIM))
    _check(ws, "ws", (S, WINDOW))
    max_nc = ck.shape[1]
    _check(ck, "ck", (S, max_nc, HEAD_DIM))
    _check(cv, "cv", (S, max_nc, HEAD_DIM))
    return S, max_nc


def cache_append(k_new: torch.Tensor, v_new: torch.Tensor, s_new: torch.Tensor,
                 ctx_len: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor, ws: torch.Tensor,
                 ck: torch.Tensor, cv: torch.Tensor) -> None:
    """Append one token per sequence to the decode cache, in place.

    k_new, v_new [S, 512]; s_new [S]; ctx_len [S] int32 (counts the new
    token); wk, wv [S, 128, 512] and ws [S, 128] rings (slot = position mod
    128); ck, cv [S, max_nc, 512]: entry L/128 - 1 is written when L is a
    multiple of 128."""
    S, max_nc = _check_append(k_new, v_new, s_new, ctx_len, wk, wv, ws, ck, cv)
    _ok("hca_cache_append", lib().hca_cache_append(
        k_new.data_ptr(), v_new.data_ptr(), s_new.data_ptr(), ctx_len.data_ptr(), S,
        wk.data_ptr(), wv.data_ptr(), ws.data_ptr(), _ptr(ck) if max_nc else None,
        _ptr(cv) if max_nc else None, max_nc, _stream(k_new.device)))


def decode_step(q: torch.Tensor, g: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                s_new: torch.Tensor, ctx_len: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor,
                ws: torch.Tensor, ck: torch.Tensor, cv: torch.Tensor,
                scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One serving step: cache_append of the new tokens, then decode of their
    queries q, g [S, 64, 512] against the updated cache."""
    S, max_nc = _check_append(k_new, v_new, s_new, ctx_len, wk, wv, ws, ck, cv)
    _check(q, "q", (S, HEADS, HEAD_DIM))
    _check(g, "g", (S, HEADS, HEAD_DIM))
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    if workspace is None:
        workspace = decode_workspace(S, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (S, HEADS, HEAD_DIM))
    _check(workspace, "workspace", dtype=torch.uint8)
    _ok("hca_decode_step", lib().hca_decode_step(
        q.data_ptr(), g.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), s_new.data_ptr(),
        ctx_len.data_ptr(), S, HEADS, ctypes.c_float(scale), wk.data_ptr(), wv.data_ptr(),
        ws.data_ptr(), _ptr(ck) if max_nc else None, _ptr(cv) if max_nc else None, max_nc,
        workspace.data_ptr(), workspace.numel(), out.data_ptr(), _stream(q.device)))
    return out


def quantize_e4m3(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """FP8 storage of bf16 rows x [..., 512]: (codes uint8 [..., 512], scale
    fp32 [...]), scale = amax / 448 per row, codes = e4m3(x / scale)."""
    if x.shape[-1] != HEAD_DIM:
        raise ValueError(f"x rows must be {HEAD_DIM} wide")
    _check(x, "x", tuple(x.shape))
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    rows = x.numel() // HEAD_DIM
    _ok("hca_quantize_e4m3", lib().hca_quantize_e4m3(
        x.data_ptr(), rows, codes.data_ptr(), scale.data_ptr(), _stream(x.device)))
    return codes, scale


def decode_e4m3(q: torch.Tensor, ck: torch.Tensor, ck_scale: torch.Tensor, cv: torch.Tensor,
                cv_scale: torch.Tensor, wk: torch.Tensor, wk_scale: torch.Tensor,
                wv: torch.Tensor, wv_scale: torch.Tensor, ctx_len: torch.Tensor, g: torch.Tensor,
                scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode step over an FP8 cache (codes and row scales from
    ``quantize_e4m3``): q, g [S, 64, 512] bf16; ck, cv [S, max_nc, 512] codes
    with [S, max_nc] scales; wk, wv [S, 128, 512] ring codes with [S, 128]
    scales; ctx_len [S] int32."""
    S, H, D = q.shape
    _check(q, "q", (S, H, HEAD_DIM))
    _check(g, "g", (S, H, HEAD_DIM))
    max_nc = ck.shape[1]
    for t, n, shp in ((ck, "ck", (S, max_nc, HEAD_DIM)), (cv, "cv", (S, max_nc, HEAD_DIM)),
                      (wk, "wk", (S, WINDOW, HEAD_DIM)), (wv, "wv", (S, WINDOW, HEAD_DIM))):
        _check(t, n, shp, dtype=torch.uint8)
    for t, n, shp in ((ck_scale, "ck_scale", (S, max_nc)), (cv_scale, "cv_scale", (S, max_nc)),
                      (wk_scale, "wk_scale", (S, WINDOW)), (wv_scale, "wv_scale", (S, WINDOW))):
        _check(t, n, shp, dtype=torch.float32)
    _check(ctx_len, "ctx_len", (S,), dtype=torch.int32)
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    if workspace is None:
        workspace = decode_workspace(S, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (S, H, HEAD_DIM))
    _check(workspace, "workspace", dtype=torch.uint8)
    _ok("hca_decode_e4m3", lib().hca_decode_e4m3(
        q.data_ptr(), _ptr(ck) if max_nc else None, _ptr(ck_scale) if max_nc else None,
        _ptr(cv) if max_nc else None, _ptr(cv_scale) if max_nc else None, max_nc,
        wk.data_ptr(), wk_scale.data_ptr(), wv.data_ptr(), wv_scale.data_ptr(),
        ctx_len.data_ptr(), g.data_ptr(), S, H, ctypes.c_float(scale), workspace.data_ptr(),
        workspace.numel(), out.data_ptr(), _stream(q.device)))
    return out


def device_error(device: Optional[torch.device] = None) -> Tuple[int, int]:
    """(status, where) from the device-side error word (synchronises the stream)."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    where = ctypes.c_uint(0)
    code = lib().hca_get_device_error(_stream(device), ctypes.byref(where))
    return code, where.value


def selftest_bounded_wait(limit_us: int, device: Optional[torch.device] = None):
    device = device or torch.device("cuda", torch.cuda.current_device())
    _ok("hca_selftest_bounded_wait", lib().hca_selftest_bounded_wait(limit_us, _stream(device)))
