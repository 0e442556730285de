"""Pins for the CPU oracle: each check ties the oracle to something other than
itself (brute force, a library routine, a closed form, a hand-derived value or
an invariant).  The last test plants mistakes in the oracle and checks that
these pins catch every one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.hca_oracle as O

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# An independent brute-force definition, written with explicit loops and
# explicit token sets (no nc formula, no vectorisation).
# ---------------------------------------------------------------------------
def brute_force(q, k, v, s, g, blk, win, scale):
    T, H, D = q.shape
    entries = []
    j = 0
    while (j + 1) * blk <= T:
        toks = list(range(j * blk, (j + 1) * blk))
        w = [math.exp(s[i]) for i in toks]
        z = sum(w)
        ck = [sum(w[n] / z * k[toks[n], d] for n in range(blk)) for d in range(D)]
        cv = [sum(w[n] / z * v[toks[n], d] for n in range(blk)) for d in range(D)]
        entries.append((toks, ck, cv))
        j += 1
    out = np.zeros((T, H, D))
    for t in range(T):
        window = [i for i in range(T) if t - win < i <= t]
        keys = [(ck, cv) for toks, ck, cv in entries if max(toks) < min(window)]
        keys += [(list(k[i]), list(v[i])) for i in window]
        for h in range(H):
            sc = [scale * sum(q[t, h, d] * kk[d] for d in range(D)) for kk, _ in keys]
            m = max(sc)
            e = [math.exp(x - m) for x in sc]
            z = sum(e)
            for d in range(D):
                o = sum(e[n] / z * keys[n][1][d] for n in range(len(keys)))
                out[t, h, d] = o / (1.0 + math.exp(-g[t, h, d]))
    return out


def rand_case(T, H, D, s_scale=1.0):
    q = RNG.standard_normal((1, T, H, D))
    k = RNG.standard_normal((1, T, D))
    v = RNG.standard_normal((1, T, D))
    s = RNG.standard_normal((1, T)) * s_scale
    g = RNG.standard_normal((1, T, H, D))
    return q, k, v, s, g


# ---- pin functions: each returns a max abs error --------------------------
def pin_brute(T=23, H=2, D=3, blk=4, win=4, seed_case=None):
    q, k, v, s, g = seed_case or rand_case(T, H, D)
    scale = 1.0 / math.sqrt(D)
    ref = brute_force(q[0], k[0], v[0], s[0], g[0], blk, win, scale)
    got = O.prefill_forward(q, k, v, s, g, blk=blk, win=win)[0]
    return float(np.abs(ref - got).max())


def sdpa_reference(q, k, v, g, mask=None, causal=False):
    qt = torch.from_numpy(q[0]).permute(1, 0, 2)[None]          # [1, H, T, D]
    H = qt.shape[1]
    kt = torch.from_numpy(k[0])[None, None].expand(1, H, -1, -1)
    vt = torch.from_numpy(v[0])[None, None].expand(1, H, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal)
    o = o[0].permute(1, 0, 2).numpy()
    return o / (1.0 + np.exp(-g[0]))


def pin_causal(T=100, H=4, D=32):
    q, k, v, s, g = rand_case(T, H, D)
    ref = sdpa_reference(q, k, v, g, causal=True)
    got = O.prefill_forward(q, k, v, s, g)[0]
    return float(np.abs(ref - got).max())


def pin_band(T=254, H=2, D=16):
    q, k, v, s, g = rand_case(T, H, D)
    t = np.arange(T)[:, None]
    i = np.arange(T)[None, :]
    mask = (i <= t) & (i > t - 128)
    ref = sdpa_reference(q, k, v, g, mask=mask)
    got = O.prefill_forward(q, k, v, s, g)[0]
    return float(np.abs(ref - got).max())


def pin_hand_avg(golden):
    T, D = 16, 1
    q = np.zeros((1, T, 1, D))
    k = np.zeros((1, T, D))
    v = np.arange(T, dtype=np.float64).reshape(1, T, D)
    s = np.zeros((1, T))
    g = np.full((1, T, 1, D), 50.0)
    got = O.prefill_forward(q, k, v, s, g, blk=4, win=4)[0, :, 0, 0]
    return max(abs(got[t] - val) for t, val in golden["avg"])


def pin_hand_nc(golden):
    return max(abs(O.num_visible_blocks(t) - n) for t, n in golden["nc"])


def pin_hand_cmp(golden):
    k = np.array([[[8.0], [16.0], [24.0], [32.0]]])
    s = np.array([[0.0, 0.0, math.log(2.0), math.log(4.0)]])
    ck, cv = O.compress(k, k, s, blk=4)
    return abs(ck[0, 0, 0] - golden["cmp"][0][0])


def pin_gate_half(T=60, H=2, D=8):
    q, k, v, s, _ = rand_case(T, H, D)
    g0 = np.zeros((1, T, H, D))
    ref = sdpa_reference(q, k, v, g0, causal=True)       # includes the 0.5 gate
    got = O.prefill_forward(q, k, v, s, g0)[0]
    ungated = O.prefill_forward(q, k, v, s, np.full_like(g0, 60.0))[0]
    return float(max(np.abs(ref - got).max(), np.abs(0.5 * ungated - got).max()))


def pin_decode_vs_prefill(T=45, H=2, D=4, blk=4, win=4, ts=None):
    q, k, v, s, g = rand_case(T, H, D)
    pre = O.prefill_forward(q, k, v, s, g, blk=blk, win=win)[0]
    ck, cv = O.compress(k, v, s, blk=blk)
    err = 0.0
    for t in (ts or range(T)):
        L = t + 1
        ring_k = np.zeros((win, D))
        ring_v = np.zeros((win, D))
        for p in range(max(0, L - win), L):
            ring_k[p % win] = k[0, p]
            ring_v[p % win] = v[0, p]
        d = O.decode_forward(q[:, t], ck, cv, ring_k[None], ring_v[None], [L], g[:, t],
                             blk=blk, win=win)
        err = max(err, float(np.abs(d[0] - pre[t]).max()))
    return err


def pin_const_block():
    D = 6
    c = RNG.standard_normal(D)
    k = np.tile(c, (1, 8, 1)).reshape(1, 8, D)
    s = RNG.standard_normal((1, 8)) * 3
    ck, cv = O.compress(k, k, s, blk=8)
    return float(np.abs(ck[0, 0] - c).max())


def pin_uniform_mean():
    k = RNG.standard_normal((2, 12, 5))
    v = RNG.standard_normal((2, 12, 5))
    s = np.full((2, 12), 0.7)
    ck, cv = O.compress(k, v, s, blk=4)
    ref_k = np.mean(k.reshape(2, 3, 4, 5), axis=2)
    ref_v = np.mean(v.reshape(2, 3, 4, 5), axis=2)
    return float(max(np.abs(ck - ref_k).max(), np.abs(cv - ref_v).max()))


ALL_PINS = {
    "brute_4_4": lambda gd: pin_brute(),
    "brute_8_8": lambda gd: pin_brute(T=37, blk=8, win=8),
    "brute_4_8": lambda gd: pin_brute(T=30, blk=4, win=8),
    "brute_8_4": lambda gd: pin_brute(T=30, blk=8, win=4),
    "causal": lambda gd: pin_causal(),
    "band": lambda gd: pin_band(),
    "hand_avg": pin_hand_avg,
    "hand_nc": pin_hand_nc,
    "hand_cmp": pin_hand_cmp,
    "gate_half": lambda gd: pin_gate_half(),
    "decode_vs_prefill": lambda gd: pin_decode_vs_prefill(),
    "const_block": lambda gd: pin_const_block(),
    "uniform_mean": lambda gd: pin_uniform_mean(),
}


@pytest.fixture(scope="module")
def golden(golden_dir):
    out = {"nc": [], "avg": [], "cmp": []}
    with open(os.path.join(golden_dir, "hand_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "nc":
                out["nc"].append((int(parts[1]), int(parts[2])))
            elif parts[0] == "avg":
                out["avg"].append((int(parts[1]), float(parts[2])))
            elif parts[0] == "cmp":
                out["cmp"].append((float(parts[1]),))
    assert out["nc"] and out["avg"] and out["cmp"]
    return out


@pytest.mark.parametrize("name", sorted(ALL_PINS))
def test_pin(name, golden):
    assert ALL_PINS[name](golden) < 1e-9, name


def test_structure_constants(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "hca_structure.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, value = line.split()[:2]
                vals[name] = int(value)
    assert vals["block_tokens"] == O.BLOCK
    assert vals["window_tokens"] == O.WINDOW
    assert vals["head_dim"] == O.HEAD_DIM
    assert vals["query_heads"] == O.HEADS


def test_brute_force_realistic_block_and_window():
    """blk = win = 128 on a ragged T: several compressed entries become
    visible, and t = 254 / 255 straddle the first step of nc."""
    case = rand_case(300, 1, 3)
    assert pin_brute(T=300, H=1, D=3, blk=128, win=128, seed_case=case) < 1e-9


def test_decode_vs_prefill_realistic():
    ts = [0, 1, 126, 127, 128, 254, 255, 256, 382, 383, 399]
    assert pin_decode_vs_prefill(T=400, H=2, D=4, blk=128, win=128, ts=ts) < 1e-9


def test_shift_invariance_of_scores():
    k = RNG.standard_normal((1, 16, 4))
    v = RNG.standard_normal((1, 16, 4))
    s = RNG.standard_normal((1, 16))
    shift = np.repeat(RNG.standard_normal(4) * 10, 4)[None]
    a = O.compress(k, v, s, blk=4)
    b = O.compress(k, v, s + shift, blk=4)
    assert np.abs(a[0] - b[0]).max() < 1e-12 and np.abs(a[1] - b[1]).max() < 1e-12


def test_one_hot_scores():
    k = RNG.standard_normal((1, 8, 4))
    s = np.zeros((1, 8))
    s[0, 5] = 60.0
    ck, cv = O.compress(k, k, s, blk=8)
    assert np.abs(ck[0, 0] - k[0, 5]).max() < 1e-20 + 8 * math.exp(-60) * 10


def test_tail_tokens_not_compressed():
    k = RNG.standard_normal((1, 10, 3))
    s = RNG.standard_normal((1, 10))
    ck, _ = O.compress(k, k, s, blk=4)
    assert ck.shape == (1, 2, 3)


def test_window_permutation_invariance():
    S, H, D, win = 1, 2, 4, 8
    q = RNG.standard_normal((S, H, D))
    g = RNG.standard_normal((S, H, D))
    ck = RNG.standard_normal((S, 5, D))
    cv = RNG.standard_normal((S, 5, D))
    wk = RNG.standard_normal((S, win, D))
    wv = RNG.standard_normal((S, win, D))
    perm = RNG.permutation(win)
    a = O.decode_forward(q, ck, cv, wk, wv, [40], g, blk=8, win=win)
    b = O.decode_forward(q, ck, cv, wk[:, perm], wv[:, perm], [40], g, blk=8, win=win)
    assert np.abs(a - b).max() < 1e-12


def test_lse_matches_definition():
    q, k, v, s, g = rand_case(20, 2, 4)
    out, lse = O.prefill_forward(q, k, v, s, g, blk=4, win=4, return_lse=True)
    # lse of a query with a single visible key (t = 0) is its scaled score.
    assert abs(lse[0, 0, 1] - q[0, 0, 1] @ k[0, 0] / 2.0) < 1e-12


def test_round_bf16_against_torch():
    x = RNG.standard_normal(1000) * 10
    ref = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(x), ref)


def test_visited_pairs_closed_form():
    # T <= 128: plain causal, T (T + 1) / 2 pairs.
    assert O.visited_pairs(100) == 100 * 101 // 2
    # counts quoted for the tiny and 32K workloads
    assert O.visited_pairs(1024) == 125639
    assert O.decode_keys([131072]) == 1023 + 128
    assert O.decode_keys([5]) == 5


# ---------------------------------------------------------------------------
# Planted mistakes: every mutant below must make at least one pin fail.
# ---------------------------------------------------------------------------
def _mutants():
    orig_nc = O.num_visible_blocks
    orig_ws = O.window_start
    orig_bw = O.block_weights
    orig_sig = O.sigmoid
    orig_attend = O.attend

    def attend_no_scale(qr, keys, values, mask, scale):
        return orig_attend(qr, keys, values, mask, 1.0)

    def attend_swapped(qr, keys, values, mask, scale):
        return orig_attend(qr, values, keys, mask, scale)

    def attend_drop_last(qr, keys, values, mask, scale):
        m = mask.copy()
        idx = np.argmax(np.cumsum(m, axis=1), axis=1)
        m[np.arange(len(m)), idx] = False
        m[:, 0] |= ~m.any(axis=1)
        return orig_attend(qr, keys, values, m, scale)

    return {
        "nc_plus_one": ("num_visible_blocks", lambda t, blk=128, win=128: orig_nc(t, blk, win) + (1 if t > win else 0)),
        "nc_uses_t_plus_1": ("num_visible_blocks", lambda t, blk=128, win=128: max(0, (t + 1) // blk)),
        "window_one_short": ("window_start", lambda t, win=128: max(0, t - win + 2)),
        "window_one_long": ("window_start", lambda t, win=128: max(0, t - win)),
        "uniform_weights": ("block_weights", lambda sb: np.full_like(sb, 1.0 / sb.shape[-1])),
        "weights_no_exp": ("block_weights", lambda sb: sb / sb.sum(-1, keepdims=True)),
        "gate_sign": ("sigmoid", lambda x: orig_sig(-x)),
        "no_gate": ("sigmoid", lambda x: np.ones_like(x)),
        "no_scale": ("attend", attend_no_scale),
        "k_v_swapped": ("attend", attend_swapped),
        "drop_newest_key": ("attend", attend_drop_last),
    }


@pytest.mark.parametrize("mutant", sorted(_mutants()))
def test_pins_catch_planted_mistake(mutant, golden, monkeypatch):
    attr, fn = _mutants()[mutant]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for name, pin in ALL_PINS.items():
        try:
            err = pin(golden)
        except Exception:  # a crash also counts as a caught mistake
            err = float("inf")
        if not err < 1e-9:
            failed.append(name)
    assert failed, f"no pin caught mutant {mutant}"
