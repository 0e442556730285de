"""Pins for the oracle's incremental cache update (``cache_append``): built
token by token from an empty cache, it must equal the whole-sequence
compressor (itself pinned to brute force and closed forms) and the directly
built raw window, and a brute-force loop on a tiny block; planted mistakes
in the update must each break the pin."""
import math

import numpy as np
import pytest

import oracle.hca_oracle as O

RNG = np.random.default_rng(77)


def build_incrementally(append, k, v, s, blk, win, max_nc):
    T, D = k.shape
    wk, wv, ws = np.zeros((win, D)), np.zeros((win, D)), np.zeros(win)
    ck, cv = np.zeros((max_nc, D)), np.zeros((max_nc, D))
    for p in range(T):
        append(wk, wv, ws, ck, cv, k[p], v[p], s[p], p + 1, blk=blk, win=win)
    return wk, wv, ws, ck, cv


def _amax(x):
    return float(np.abs(x).max()) if x.size else 0.0


def pin_error(append, T=700, D=8, blk=128):
    """Max abs difference between the incrementally built cache and the
    definition (whole-sequence compression + directly placed ring)."""
    k = RNG.standard_normal((T, D))
    v = RNG.standard_normal((T, D))
    s = RNG.standard_normal(T) * 2.0
    nb = T // blk
    wk, wv, ws, ck, cv = build_incrementally(append, k, v, s, blk, blk, nb + 1)
    rck, rcv = O.compress(k[None], v[None], s[None], blk)
    err = max(_amax(ck[:nb] - rck[0]), _amax(cv[:nb] - rcv[0]),
              _amax(ck[nb:]), _amax(cv[nb:]))   # nothing past the last complete block
    ring_k = np.zeros((blk, D))
    ring_v = np.zeros((blk, D))
    ring_s = np.zeros(blk)
    for p in range(max(0, T - blk), T):
        ring_k[p % blk], ring_v[p % blk], ring_s[p % blk] = k[p], v[p], s[p]
    return max(err, _amax(wk - ring_k), _amax(wv - ring_v), _amax(ws - ring_s))


def test_incremental_equals_whole_sequence_compression():
    for T in (1, 127, 128, 129, 700):
        assert pin_error(O.cache_append, T=T) < 1e-12, T


def test_tiny_block_brute_force():
    """blk = win = 4: entry j by explicit loops over the block's tokens."""
    T, D, blk = 11, 3, 4
    k = RNG.standard_normal((T, D))
    v = RNG.standard_normal((T, D))
    s = RNG.standard_normal(T)
    _, _, _, ck, cv = build_incrementally(O.cache_append, k, v, s, blk, blk, 3)
    for j in range(T // blk):
        toks = range(j * blk, (j + 1) * blk)
        w = [math.exp(s[i]) for i in toks]
        z = sum(w)
        for d in range(D):
            assert abs(ck[j, d] - sum(w[n] / z * k[i, d] for n, i in enumerate(toks))) < 1e-12
            assert abs(cv[j, d] - sum(w[n] / z * v[i, d] for n, i in enumerate(toks))) < 1e-12


def test_ring_must_hold_one_block():
    with pytest.raises(ValueError):
        O.cache_append(np.zeros((8, 2)), np.zeros((8, 2)), np.zeros(8), np.zeros((2, 2)),
                       np.zeros((2, 2)), np.zeros(2), np.zeros(2), 0.0, 4, blk=4, win=8)


# ---- planted mistakes -------------------------------------------------------
def _slot_off_by_one(wk, wv, ws, ck, cv, k_new, v_new, s_new, L, blk=128, win=128):
    slot = L % win
    wk[slot], wv[slot], ws[slot] = k_new, v_new, s_new
    if L % blk == 0:
        w = O.block_weights(ws)
        ck[L // blk - 1], cv[L // blk - 1] = w @ wk, w @ wv


def _compress_before_write(wk, wv, ws, ck, cv, k_new, v_new, s_new, L, blk=128, win=128):
    if L % blk == 0:
        w = O.block_weights(ws)
        ck[L // blk - 1], cv[L // blk - 1] = w @ wk, w @ wv
    slot = (L - 1) % win
    wk[slot], wv[slot], ws[slot] = k_new, v_new, s_new


def _entry_index_shifted(wk, wv, ws, ck, cv, k_new, v_new, s_new, L, blk=128, win=128):
    slot = (L - 1) % win
    wk[slot], wv[slot], ws[slot] = k_new, v_new, s_new
    if L % blk == 0 and L // blk < len(ck):
        w = O.block_weights(ws)
        ck[L // blk], cv[L // blk] = w @ wk, w @ wv


def _k_weights_for_v(wk, wv, ws, ck, cv, k_new, v_new, s_new, L, blk=128, win=128):
    slot = (L - 1) % win
    wk[slot], wv[slot], ws[slot] = k_new, v_new, s_new
    if L % blk == 0:
        w = O.block_weights(ws)
        ck[L // blk - 1], cv[L // blk - 1] = w @ wk, w @ wk


@pytest.mark.parametrize("mutant", [_slot_off_by_one, _compress_before_write,
                                    _entry_index_shifted, _k_weights_for_v])
def test_pin_catches_planted_mistake(mutant):
    try:
        err = pin_error(mutant, T=300)
    except Exception:   # a crash also counts as caught
        err = float("inf")
    assert not err < 1e-9, mutant.__name__
