"""Seeded synthetic inputs for the HCA workloads.

This module holds no attention arithmetic: it only draws N(0, 1) numbers and
lays them out.  Both the CUDA path (tests, bench) and the CPU oracle receive
their inputs from here, so the two sides see bit-identical bf16 tensors.

Recipe.  Every tensor is drawn in chunks of ``CHUNK`` rows.  Chunk c of tensor
`name` under base seed b uses its own ``torch.Generator('cpu')`` seeded with
``chunk_seed(b, name, c)``; the chunk is drawn as float32 ``randn`` and rounded
to bfloat16 (round to nearest even).  Independent chunks let the host draw
them on many threads and let a test regenerate only the chunks that hold the
rows it samples.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

HEADS = 64
HEAD_DIM = 512
BLOCK = 128
WINDOW = 128
CHUNK = 1024

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "s": 4, "g": 5, "ck": 6, "cv": 7, "wk": 8, "wv": 9,
               "vha_down": 10, "vha_up": 11, "dout": 12}
_MASK63 = (1 << 63) - 1


def chunk_seed(base: int, name: str, chunk: int) -> int:
    """Deterministic 63-bit seed for one chunk of one tensor."""
    x = (base * 0x9E3779B97F4A7C15 + _TENSOR_IDS[name] * 0xBF58476D1CE4E5B9
         + chunk * 0x94D049BB133111EB + 0x2545F4914F6CDD1D) & _MASK63
    x ^= x >> 31
    x = (x * 0xD6E8FEB86659FD93) & _MASK63
    x ^= x >> 29
    return x


def _threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(n, 64))


def _draw_chunk(base: int, name: str, c: int, rows: int, row_shape, scale: float):
    g = torch.Generator("cpu").manual_seed(chunk_seed(base, name, c))
    x = torch.randn((rows, *row_shape), generator=g, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def normal_bf16(base: int, name: str, rows: int, row_shape: Sequence[int] = (),
                scale: float = 1.0, chunks: Optional[Sequence[int]] = None,
                pin: bool = False) -> torch.Tensor:
    """bf16 tensor [rows, *row_shape] of N(0, 1) draws (times `scale`, applied
    in float32 before rounding; 0.5 is exact).  With `chunks`, only those
    chunk indices are drawn and the rest of the tensor is zero."""
    row_shape = tuple(row_shape)
    out = torch.empty((rows, *row_shape), dtype=torch.bfloat16, pin_memory=pin)
    nchunks = (rows + CHUNK - 1) // CHUNK
    todo = range(nchunks) if chunks is None else sorted(set(chunks))
    if chunks is not None:
        out.zero_()

    def work(c):
        r0 = c * CHUNK
        r1 = min(rows, r0 + CHUNK)
        out[r0:r1] = _draw_chunk(base, name, c, r1 - r0, row_shape, scale)

    prev = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, todo))
    finally:
        torch.set_num_threads(prev)
    return out


def chunk_rows(base: int, name: str, c: int, rows: int, row_shape: Sequence[int] = (),
               scale: float = 1.0) -> torch.Tensor:
    """Rows [c * CHUNK, min(rows, (c + 1) * CHUNK)) of the tensor that
    ``normal_bf16(base, name, rows, row_shape, scale)`` draws, without drawing
    the rest (same generator, same values)."""
    r0 = c * CHUNK
    r1 = min(rows, r0 + CHUNK)
    return _draw_chunk(base, name, c, r1 - r0, tuple(row_shape), scale)


# ---------------------------------------------------------------------------
# Workload definitions
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    T: int
    seed: int
    k_scale: float = 1.0


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    S: int
    seed: int
    ctx: Optional[int] = None          # fixed context length for every sequence
    ctx_lo: Optional[int] = None       # else drawn uniformly in [ctx_lo, ctx_hi]
    ctx_hi: Optional[int] = None
    from_raw: bool = True              # cache built by compressing raw K/V/s


PREFILL_TINY = PrefillConfig("prefill_T1024", B=1, T=1024, seed=0)
PREFILL_32K = PrefillConfig("prefill_T32768_kx0.5", B=1, T=32768, seed=1, k_scale=0.5)
PREFILL_128K = PrefillConfig("prefill_T131072", B=1, T=131072, seed=2)
DECODE_64x128K = DecodeConfig("decode_S64_L131072", S=64, seed=3, ctx=131072, from_raw=True)
DECODE_16xLONG = DecodeConfig("decode_S16_L64K-1M", S=16, seed=4, ctx_lo=65536, ctx_hi=1048576,
                              from_raw=False)

CONFIGS = [PREFILL_TINY, PREFILL_32K, PREFILL_128K, DECODE_64x128K, DECODE_16xLONG]


def prefill_inputs(cfg: PrefillConfig, chunks: Optional[Sequence[int]] = None,
                   pin: bool = False):
    """dict of CPU bf16 tensors q, g [B, T, H, D]; k, v [B, T, D]; s [B, T].

    `chunks` restricts q and g to the token chunks listed (the rest zero);
    k, v and s are always drawn in full.  Batch b uses base seed
    ``cfg.seed * 1000 + b``.
    """
    B, T = cfg.B, cfg.T
    out = {n: [] for n in ("q", "k", "v", "s", "g")}
    for b in range(B):
        base = cfg.seed * 1000 + b
        out["q"].append(normal_bf16(base, "q", T, (HEADS, HEAD_DIM), chunks=chunks, pin=pin))
        out["k"].append(normal_bf16(base, "k", T, (HEAD_DIM,), scale=cfg.k_scale, pin=pin))
        out["v"].append(normal_bf16(base, "v", T, (HEAD_DIM,), pin=pin))
        out["s"].append(normal_bf16(base, "s", T, (), pin=pin))
        out["g"].append(normal_bf16(base, "g", T, (HEADS, HEAD_DIM), chunks=chunks, pin=pin))
    return {n: torch.stack(v) if B > 1 else v[0].unsqueeze(0) for n, v in out.items()}


def decode_ctx_lens(cfg: DecodeConfig) -> List[int]:
    if cfg.ctx is not None:
        return [cfg.ctx] * cfg.S
    g = torch.Generator("cpu").manual_seed(cfg.seed)
    return [int(x) for x in torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (cfg.S,), generator=g)]


def decode_raw_sequence(cfg: DecodeConfig, seq: int, L: int):
    """Raw K, V [L, D] and scores s [L] of one decode sequence (from_raw)."""
    base = cfg.seed * 1000 + seq
    k = normal_bf16(base, "k", L, (HEAD_DIM,))
    v = normal_bf16(base, "v", L, (HEAD_DIM,))
    s = normal_bf16(base, "s", L, ())
    return k, v, s


def ring_window(raw: torch.Tensor, L: int, win: int = WINDOW) -> torch.Tensor:
    """Place the newest min(L, win) rows of `raw` [>=L, D] into a ring buffer
    [win, D]: the token at position p goes to slot p mod win; unused slots 0."""
    D = raw.shape[-1]
    ring = torch.zeros((win, D), dtype=raw.dtype)
    p0 = max(0, L - win)
    for p in range(p0, L):
        ring[p % win] = raw[p]
    return ring


def decode_direct_sequence(cfg: DecodeConfig, seq: int, max_nc: int):
    """Cache entries and window drawn directly as N(0, 1) (no raw tokens):
    ck, cv [max_nc, D] and wk, wv [WINDOW, D].  Every row is drawn, including
    rows the sequence's context length leaves unused."""
    base = cfg.seed * 1000 + seq
    ck = normal_bf16(base, "ck", max_nc, (HEAD_DIM,))
    cv = normal_bf16(base, "cv", max_nc, (HEAD_DIM,))
    wk = normal_bf16(base, "wk", WINDOW, (HEAD_DIM,))
    wv = normal_bf16(base, "wv", WINDOW, (HEAD_DIM,))
    return ck, cv, wk, wv


def vha_factors(rank: int, seed: int, scale: float = 1.0 / 16):
    """Virtual-head-attention factors (down, up), each [64, rank] bf16, drawn
    N(0, scale^2).  The default 1/16 (a light mix) makes the mixed-in term
    about sqrt(rank)/32 of the size of the gated output."""
    return (normal_bf16(seed, "vha_down", HEADS, (rank,), scale),
            normal_bf16(seed, "vha_up", HEADS, (rank,), scale))


def decode_query(cfg: DecodeConfig):
    """q, g [S, H, D] for one decode step."""
    base = cfg.seed * 1000 + 999
    q = normal_bf16(base, "q", cfg.S, (HEADS, HEAD_DIM))
    g = normal_bf16(base, "g", cfg.S, (HEADS, HEAD_DIM))
    return q, g
