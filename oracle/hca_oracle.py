"""Plain fp64 CPU oracle for Heavily Compressed Attention (HCA).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library; it is deliberately slow and written so that each
step can be checked against the pages by eye.

What the pages say (all prose, no equations):

* 'BaiduがERNIE 5.5 Flash Baseを公開' (hackernews.jp), §2.1 Latent-Gated Sparse
  Attention, and its Chinese twin 'ERNIE 5.5 Flash Base 正式发布' §2.1: an HCA
  layer turns every 128 tokens into one cache entry and runs dense attention
  over all of those entries plus a short window of recent uncompressed tokens;
  HCA heads are 512 wide for query/key and value; the model has 64 attention
  heads; every layer multiplies its attention output by a learned gate.
* xenospectrum, 'ERNIE 5.5 Flash Base' analysis, section 活性140億パラメータと
  長文処理を支える仕組み: the window is the most recent 128 tokens, kept
  uncompressed as a sliding window.

Readings adopted where the pages are silent (each is listed with its reason in
the design notes of the repository):

* one shared KV head; the compressor of block j is the within-block
  softmax(s)-weighted sum of the block's K rows and, with the same weights, of
  its V rows, where s is a per-token scalar score input;
* query t sees compressed entry j only if block j lies wholly before its
  window, i.e. j < nc(t) = max(0, floor((t - W + 1) / blk)), and the raw keys
  max(0, t - W + 1) .. t (the window includes the query token itself);
* one softmax over the union of both key sets, one scale 1/sqrt(D) for all
  keys, no positional encoding, no sink;
* out = sigmoid(g) * o, elementwise over [T, H, D];
* virtual head attention, when asked for, mixes the heads of each position's
  gated output: y = x + up (down^T x) with down, up [H, r].

Parity status: pinned.  The tests under ``tests/test_oracle_pins.py`` tie
every function here to something other than itself: a brute-force loop
implementation with an explicitly built key list and mask; PyTorch's fp64
``scaled_dot_product_attention`` for the cases that reduce to causal and
banded attention; closed forms (constant block, uniform scores, gate at 0,
hand-derived golden values); invariants (shift, permutation); and decode vs
prefill agreement.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

HEADS = 64
HEAD_DIM = 512
BLOCK = 128
WINDOW = 128


# ---------------------------------------------------------------------------
# Visibility rule
# ---------------------------------------------------------------------------
def window_start(t: int, win: int = WINDOW) -> int:
    """First raw key of query t's window: the last `win` tokens up to and
    including t (xenospectrum analysis, 活性140億パラメータと長文処理を支える
    仕組み: the newest 128 tokens stay uncompressed)."""
    return max(0, t - win + 1)


def num_visible_blocks(t: int, blk: int = BLOCK, win: int = WINDOW) -> int:
    """nc(t): how many compressed entries query t sees.

    Block j covers tokens blk*j .. blk*j + blk - 1.  It is visible when it lies
    wholly before the window, i.e. blk*(j+1) <= t - win + 1.  Counting the j
    that satisfy this gives floor((t - win + 1) / blk), clamped at 0.
    ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1: entries for every 128 tokens,
    plus a short raw window.)
    """
    return max(0, (t - win + 1) // blk)


# ---------------------------------------------------------------------------
# Compressor
# ---------------------------------------------------------------------------
def block_weights(s_block: np.ndarray) -> np.ndarray:
    """softmax over the tokens of one block (last axis), max-subtracted."""
    z = s_block - s_block.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def compress(k: np.ndarray, v: np.ndarray, s: np.ndarray, blk: int = BLOCK):
    """Compressed cache entries for every complete block.

    k, v: [B, T, D]; s: [B, T].  Returns cK, cV: [B, T // blk, D] in fp64.
    Entry j = sum_i softmax(s[blk*j : blk*j+blk])_i * row_i.  Tokens of a
    trailing partial block are not compressed.
    ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1: 128 tokens -> 1 cache entry.)
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    B, T, D = k.shape
    nb = T // blk
    kb = k[:, : nb * blk].reshape(B, nb, blk, D)
    vb = v[:, : nb * blk].reshape(B, nb, blk, D)
    w = block_weights(s[:, : nb * blk].reshape(B, nb, blk))
    ck = np.einsum("bni,bnid->bnd", w, kb)
    cv = np.einsum("bni,bnid->bnd", w, vb)
    return ck, cv


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as
    fp64.  Used only by the optional diagnosis mode that mimics a bf16 cache."""
    f32 = np.asarray(x, dtype=np.float32)
    bits = f32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32)
    nan = np.isnan(f32)
    out = np.where(nan, f32, out)
    return out.astype(np.float64)


# ---------------------------------------------------------------------------
# Attention core
# ---------------------------------------------------------------------------
def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def vha_mix(x: np.ndarray, down: np.ndarray, up: np.ndarray) -> np.ndarray:
    """Virtual head attention: after attention, a light low-rank mix across the
    heads of one position, with an identity skip ('BaiduがERNIE 5.5 Flash Base
    を公開' §2.1, virtual head attention; 'ERNIE 5.5 Flash Base 正式发布' §2.1,
    VHA).  The pages give neither the rank nor where the gate sits; the
    reading here: the mix acts on the gated output of each position,

        y[h] = x[h] + sum_r up[h, r] * sum_k down[k, r] * x[k],

    x [..., H, D] (heads on the second-to-last axis), down and up [H, r].
    """
    x = np.asarray(x, dtype=np.float64)
    down = np.asarray(down, dtype=np.float64)
    up = np.asarray(up, dtype=np.float64)
    z = np.einsum("kr,...kd->...rd", down, x)      # [..., r, D]: the rank-r summary
    return x + np.einsum("hr,...rd->...hd", up, z)


def attend(qrows: np.ndarray, keys: np.ndarray, values: np.ndarray,
           mask: np.ndarray, scale: float):
    """Dense masked softmax attention, all heads sharing one key/value set.

    qrows: [n, H, D]; keys, values: [K, D]; mask: [n, K] (True = visible).
    Returns o: [n, H, D] (normalised, ungated) and lse: [n, H] (natural log of
    the softmax denominator of the scaled scores).
    """
    z = np.einsum("nhd,kd->nhk", qrows, keys) * scale
    z = np.where(mask[:, None, :], z, -np.inf)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    den = e.sum(axis=-1, keepdims=True)
    o = np.einsum("nhk,kd->nhd", e / den, values)
    lse = (m + np.log(den))[..., 0]
    return o, lse


def _prefill_rows(qrows, grows, kb, vb, ckb, cvb, positions: np.ndarray,
                  blk: int, win: int, scale: float):
    """Outputs for the given query positions of one sequence; qrows, grows
    [len(positions), H, D] are the query and gate rows of those positions.

    The key set is the union over these positions: the compressed entries
    0 .. max nc - 1 and the raw tokens from the earliest window start to the
    last position; the per-row mask then selects each query's own keys.
    """
    t_lo, t_hi = int(positions.min()), int(positions.max())
    n_c = num_visible_blocks(t_hi, blk, win)
    r0 = window_start(t_lo, win)
    keys = np.concatenate([ckb[:n_c], kb[r0 : t_hi + 1]], axis=0)
    vals = np.concatenate([cvb[:n_c], vb[r0 : t_hi + 1]], axis=0)
    raw_idx = np.arange(r0, t_hi + 1)
    ent_idx = np.arange(n_c)
    mask = np.zeros((len(positions), n_c + len(raw_idx)), dtype=bool)
    for row, t in enumerate(positions):
        t = int(t)
        mask[row, :n_c] = ent_idx < num_visible_blocks(t, blk, win)
        mask[row, n_c:] = (raw_idx >= window_start(t, win)) & (raw_idx <= t)
    o, lse = attend(qrows, keys, vals, mask, scale)
    out = sigmoid(grows) * o
    return out, lse


def prefill_forward(q, k, v, s, g, blk: int = BLOCK, win: int = WINDOW,
                    scale: Optional[float] = None,
                    positions: Optional[Sequence[int]] = None,
                    round_cache_bf16: bool = False, chunk: int = 128,
                    return_lse: bool = False, cache=None, rows_only: bool = False,
                    vha=None):
    """HCA prefill forward in fp64.

    q, g: [B, T, H, D]; k, v: [B, T, D]; s: [B, T].  Returns out [B, T, H, D]
    (or [B, len(positions), H, D] when `positions` selects rows), and the lse
    [.., H] when asked.  With ``rows_only`` q and g hold just the selected rows
    ([B, len(positions), H, D], in the order of `positions`).  `cache` may pass
    precomputed (cK, cV) from ``compress``.  `vha` = (down, up) applies
    ``vha_mix`` to the gated output of every position.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, D = k.shape
    H = q.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    ck, cv = cache if cache is not None else compress(k, v, s, blk)
    if round_cache_bf16:
        ck, cv = round_bf16(ck), round_bf16(cv)
    pos = np.arange(T) if positions is None else np.asarray(list(positions), dtype=np.int64)
    out = np.empty((B, len(pos), H, D), dtype=np.float64)
    lse = np.empty((B, len(pos), H), dtype=np.float64)
    # group the requested rows so that every group lies inside one `chunk`-long
    # stretch of positions (keeps each group's key set short)
    order = np.argsort(pos, kind="stable")
    groups = []
    start = 0
    for n in range(1, len(order) + 1):
        if n == len(order) or pos[order[n]] // chunk != pos[order[start]] // chunk:
            groups.append(order[start:n])
            start = n
    for b in range(B):
        for idx in groups:
            sel = pos[idx]
            rows = idx if rows_only else sel
            qr = np.asarray(q[b][rows], dtype=np.float64)
            gr = np.asarray(g[b][rows], dtype=np.float64)
            o, l = _prefill_rows(qr, gr, k[b], v[b], ck[b], cv[b], sel, blk, win, scale)
            out[b, idx] = o if vha is None else vha_mix(o, *vha)
            lse[b, idx] = l
    return (out, lse) if return_lse else out


def decode_forward(q, ck, cv, wk, wv, ctx_len, g, blk: int = BLOCK,
                   win: int = WINDOW, scale: Optional[float] = None,
                   return_lse: bool = False, vha=None):
    """HCA decode for one new token per sequence, in fp64.

    q, g: [S, H, D]; ck, cv: [S, max_nc, D]; wk, wv: [S, win, D] hold the
    window as a ring, the token at position p in slot p mod win; ctx_len[s] = L
    counts the new token, so the query sits at t = L - 1.  Keys are the
    compressed entries j < nc(L - 1) and the min(L, win) newest raw tokens
    (slots 0 .. L-1 when L < win, all slots otherwise).  `vha` = (down, up)
    applies ``vha_mix`` to each sequence's gated output.
    """
    q = np.asarray(q, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    ck = np.asarray(ck, dtype=np.float64)
    cv = np.asarray(cv, dtype=np.float64)
    wk = np.asarray(wk, dtype=np.float64)
    wv = np.asarray(wv, dtype=np.float64)
    S, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.empty((S, H, D), dtype=np.float64)
    lse = np.empty((S, H), dtype=np.float64)
    for si in range(S):
        L = int(ctx_len[si])
        t = L - 1
        n_c = num_visible_blocks(t, blk, win)
        n_w = min(L, win)
        keys = np.concatenate([ck[si, :n_c], wk[si, :n_w]], axis=0)
        vals = np.concatenate([cv[si, :n_c], wv[si, :n_w]], axis=0)
        mask = np.ones((1, keys.shape[0]), dtype=bool)
        o, l = attend(q[si][None], keys, vals, mask, scale)
        out[si] = sigmoid(g[si]) * o[0]
        if vha is not None:
            out[si] = vha_mix(out[si], *vha)
        lse[si] = l[0]
    return (out, lse) if return_lse else out


# ---------------------------------------------------------------------------
# Backward (training at 128K: 'BaiduがERNIE 5.5 Flash Baseを公開' §3)
# ---------------------------------------------------------------------------
def prefill_backward(q, k, v, s, g, dout, blk: int = BLOCK, win: int = WINDOW,
                     scale: Optional[float] = None, chunk: int = 128):
    """Gradients of L = sum(dout * out) for out = prefill_forward(q, k, v, s, g).

    Returns dq, dk, dv, ds, dg (the shapes of q, k, v, s, g), in fp64.  The
    steps follow the forward in reverse, one chunk of query positions at a
    time over the chunk's union key set with the per-row mask:

      out = sigmoid(g) o            dg = dout o sigmoid(g) (1 - sigmoid(g)),
                                    dO = dout sigmoid(g)
      o = P values                  dP = dO . value_j,  dvalue_j += P_j dO
      P = softmax(z) (masked)       dz = P (dP - sum_j P_j dP_j)
      z = scale q . key_j           dq = scale sum_j dz_j key_j,
                                    dkey_j += scale dz_j q
    Key j is a compressed entry or a raw token; the gradients of the entries
    then flow through the compressor of each block (softmax weights w of the
    block's scores):
      cK = sum_i w_i K_i            dK_i += w_i dcK,  dV_i += w_i dcV
      w = softmax(s_block)          ds_i = w_i (a_i - sum_m w_m a_m),
                                    a_i = dcK . K_i + dcV . V_i
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, T, D = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    ck, cv = compress(k, v, s, blk)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dg = np.zeros_like(g)
    dck = np.zeros_like(ck)
    dcv = np.zeros_like(cv)
    for b in range(B):
        for t_lo in range(0, T, chunk):
            t_hi = min(T, t_lo + chunk) - 1
            pos = np.arange(t_lo, t_hi + 1)
            n_c = num_visible_blocks(t_hi, blk, win)
            r0 = window_start(t_lo, win)
            keys = np.concatenate([ck[b, :n_c], k[b, r0 : t_hi + 1]], axis=0)
            vals = np.concatenate([cv[b, :n_c], v[b, r0 : t_hi + 1]], axis=0)
            raw_idx = np.arange(r0, t_hi + 1)
            ent_idx = np.arange(n_c)
            mask = np.zeros((len(pos), n_c + len(raw_idx)), dtype=bool)
            for row, t in enumerate(pos):
                t = int(t)
                mask[row, :n_c] = ent_idx < num_visible_blocks(t, blk, win)
                mask[row, n_c:] = (raw_idx >= window_start(t, win)) & (raw_idx <= t)
            qr = q[b, t_lo : t_hi + 1]
            z = np.einsum("nhd,kd->nhk", qr, keys) * scale
            z = np.where(mask[:, None, :], z, -np.inf)
            e = np.exp(z - z.max(axis=-1, keepdims=True))
            P = e / e.sum(axis=-1, keepdims=True)
            o = np.einsum("nhk,kd->nhd", P, vals)
            sg = sigmoid(g[b, t_lo : t_hi + 1])
            do = dout[b, t_lo : t_hi + 1]
            dg[b, t_lo : t_hi + 1] = do * o * sg * (1.0 - sg)
            dO = do * sg
            dP = np.einsum("nhd,kd->nhk", dO, vals)
            dz = P * (dP - (P * dP).sum(axis=-1, keepdims=True))
            dq[b, t_lo : t_hi + 1] = scale * np.einsum("nhk,kd->nhd", dz, keys)
            dkeys = scale * np.einsum("nhk,nhd->kd", dz, qr)
            dvals = np.einsum("nhk,nhd->kd", P, dO)
            dck[b, :n_c] += dkeys[:n_c]
            dcv[b, :n_c] += dvals[:n_c]
            dk[b, r0 : t_hi + 1] += dkeys[n_c:]
            dv[b, r0 : t_hi + 1] += dvals[n_c:]
    ds = np.zeros_like(s)
    nb = T // blk
    for b in range(B):
        for j in range(nb):
            sl = slice(j * blk, (j + 1) * blk)
            w = block_weights(s[b, sl])
            dk[b, sl] += w[:, None] * dck[b, j]
            dv[b, sl] += w[:, None] * dcv[b, j]
            a = k[b, sl] @ dck[b, j] + v[b, sl] @ dcv[b, j]
            ds[b, sl] = w * (a - (w * a).sum())
    return dq, dk, dv, ds, dg


# ---------------------------------------------------------------------------
# Incremental cache update (serving)
# ---------------------------------------------------------------------------
def cache_append(wk, wv, ws, ck, cv, k_new, v_new, s_new, L: int,
                 blk: int = BLOCK, win: int = WINDOW) -> None:
    """One serving step of one sequence's decode cache, in place (fp64 arrays).

    wk, wv: [win, D] and ws: [win] hold the raw window as a ring (token at
    position p in slot p mod win); ck, cv: [max_nc, D] the compressed entries.
    The new token sits at position p = L - 1: it is written to slot p mod win.
    When L is a multiple of blk, block j = L // blk - 1 has just completed, and
    with win == blk the ring then holds exactly that block, so entry j is the
    block's softmax(s)-weighted sum taken from the ring ('BaiduがERNIE 5.5
    Flash Baseを公開' §2.1: one cache entry per 128 tokens; xenospectrum
    analysis: the newest 128 tokens stay raw).
    """
    if win != blk:
        raise ValueError("the ring holds one whole block only when win == blk")
    slot = (L - 1) % win
    wk[slot] = k_new
    wv[slot] = v_new
    ws[slot] = s_new
    if L % blk == 0:
        j = L // blk - 1
        w = block_weights(np.asarray(ws, dtype=np.float64))
        ck[j] = w @ np.asarray(wk, dtype=np.float64)
        cv[j] = w @ np.asarray(wv, dtype=np.float64)


# ---------------------------------------------------------------------------
# FP8 (e4m3) cache storage
# ---------------------------------------------------------------------------
# The pages train with FP8 mixed precision and ship FP8 weights ('Baiduが
# ERNIE 5.5 Flash Baseを公開' §3 and §5); the decode cache can be stored the
# same way.  Reading adopted: every 512-wide cache row is stored as e4m3
# codes with one fp32 scale, scale = amax(|row|) / 448 (1 for an all-zero
# row), code = e4m3(row / scale) rounded to nearest even, saturating at the
# largest finite magnitude 448.  The row's value is code * scale.  The
# division and the rounding decision are taken in fp32, the precision the
# kernel takes them in, so both sides produce the same codes.
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 code (1 sign bit, 4 exponent bits with bias 7, 3
    mantissa bits; exponent field 0 holds subnormals m * 2^-9; 0x7F / 0xFF
    are NaN; there are no infinities).  Returned as fp64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """Round each (fp32) value to the nearest e4m3 value, ties to the even
    mantissa, magnitudes above 448 saturating to 448; NaN -> 0x7F."""
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.abs(y)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    # quantum of a's binade: 2^(e - 3) with e = floor(log2 a), at least the
    # subnormal quantum 2^-9 (binade of 2^-6 and below)
    _, ex = np.frexp(np.maximum(a, 2.0 ** -6))
    q = 2.0 ** (ex - 1 - 3)
    v = np.round(a / q) * q          # numpy rounds halves to even
    v = np.minimum(v, E4M3_MAX)
    _, ev = np.frexp(np.where(v > 0, v, 1.0))
    E = ev - 1 + 7                   # biased exponent of a normal value
    normal = v >= 2.0 ** -6
    mant_n = np.where(normal, v / 2.0 ** (ev - 1) * 8 - 8, 0)
    code = np.where(normal, (E << 3) + mant_n.astype(np.int64),
                    (v / 2.0 ** -9).astype(np.int64))
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def quantize_e4m3_rows(x: np.ndarray):
    """Per-row e4m3 storage of x [..., D]: (codes uint8 [..., D], scale fp32
    [...]) with scale = amax / 448 in fp32 and codes = e4m3(x / scale), the
    division in fp32."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.abs(x32).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x32 / scale[..., None]).astype(np.float32)
    return e4m3_encode(y), scale


def dequantize_e4m3_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """fp64 value of each stored row: code value * row scale."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


# ---------------------------------------------------------------------------
# Work counts (used for FLOP accounting and by the tests)
# ---------------------------------------------------------------------------
def visited_pairs(T: int, blk: int = BLOCK, win: int = WINDOW) -> int:
    """Number of (query, key) pairs one head visits over a sequence of T
    tokens: sum over t of nc(t) + min(t + 1, win)."""
    return sum(num_visible_blocks(t, blk, win) + (t - window_start(t, win) + 1)
               for t in range(T))


def decode_keys(ctx_len: Iterable[int], blk: int = BLOCK, win: int = WINDOW) -> int:
    """Keys visited by one decode call: sum over sequences of nc(L-1) + min(L, win)."""
    return sum(num_visible_blocks(int(L) - 1, blk, win) + min(int(L), win) for L in ctx_len)
