"""Full-output parity of large prefill workloads against the fp64 oracle.

The oracle is single-threaded NumPy; the full 32K and 128K outputs are
checked by running it on every 1024-position chunk in a pool of worker
processes, one per host core.  The pool is started with ``spawn`` (a process
forked after CUDA initialisation can hang).  Workers draw their own inputs
from the seeded generators (the same values the GPU got: ``inputs`` is the
only module both sides share) and build the fp64 compressed cache once each;
the parent sends each chunk of the GPU output and receives error sums, so the
whole output is compared element by element without ever holding it in fp64.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from typing import Dict

import numpy as np

_W: Dict = {}


def _cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _init_worker(cfg, root):
    import sys
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch
    torch.set_num_threads(1)
    from compressed_sliding_window_b200 import inputs as I
    from oracle import hca_oracle as O
    base = cfg.seed * 1000
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    k = f64(I.normal_bf16(base, "k", cfg.T, (512,), scale=cfg.k_scale))[None]
    v = f64(I.normal_bf16(base, "v", cfg.T, (512,)))[None]
    s = f64(I.normal_bf16(base, "s", cfg.T, ()))[None]
    _W.update(cfg=cfg, k=k, v=v, s=s, cache=O.compress(k, v, s), I=I, O=O, base=base)


def _check_chunk(c: int, got: np.ndarray):
    """Oracle rows of position chunk c vs the GPU rows `got` [n, 64, 512]
    (float32 copies of the bf16 output).  Returns (max_abs, sum sq diff,
    sum sq ref, all finite)."""
    cfg, I, O = _W["cfg"], _W["I"], _W["O"]
    T = cfg.T
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    q = f64(I.chunk_rows(_W["base"], "q", c, T, (64, 512)))[None]
    g = f64(I.chunk_rows(_W["base"], "g", c, T, (64, 512)))[None]
    pos = list(range(c * I.CHUNK, c * I.CHUNK + q.shape[1]))
    ref = O.prefill_forward(q, _W["k"], _W["v"], _W["s"], g, positions=pos, rows_only=True,
                            cache=_W["cache"])[0]
    got = got.astype(np.float64)
    d = got - ref
    return (float(np.abs(d).max()), float((d * d).sum()), float((ref * ref).sum()),
            bool(np.isfinite(got).all()))


def prefill_full_errors(cfg, out_gpu, workers: int = 0):
    """Compare every row of the GPU prefill output `out_gpu` [1, T, 64, 512]
    (a CUDA tensor) with the oracle.  Returns (max_abs, rel_l2, all_finite)."""
    from compressed_sliding_window_b200 import inputs as I
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    T = cfg.T
    nch = (T + I.CHUNK - 1) // I.CHUNK
    n = workers or min(_cores(), nch)
    ctx = mp.get_context("spawn")
    env_keep = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "MKL_NUM_THREADS",
                                               "OPENBLAS_NUM_THREADS")}
    for k in env_keep:
        os.environ[k] = "1"
    try:
        pool = ctx.Pool(n, initializer=_init_worker, initargs=(cfg, root))
    finally:
        for k, v in env_keep.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    max_abs, sdd, srr, finite = 0.0, 0.0, 0.0, True
    try:
        pending = []
        for c in range(nch):
            r0, r1 = c * I.CHUNK, min(T, (c + 1) * I.CHUNK)
            got = out_gpu[0, r0:r1].float().cpu().numpy()
            pending.append(pool.apply_async(_check_chunk, (c, got)))
            if len(pending) >= 2 * n:
                a, b, r, f = pending.pop(0).get()
                max_abs, sdd, srr, finite = max(max_abs, a), sdd + b, srr + r, finite and f
        for p in pending:
            a, b, r, f = p.get()
            max_abs, sdd, srr, finite = max(max_abs, a), sdd + b, srr + r, finite and f
    finally:
        pool.close()
        pool.join()
    rel = float(np.sqrt(sdd / srr)) if srr > 0 else 0.0
    return max_abs, rel, finite
