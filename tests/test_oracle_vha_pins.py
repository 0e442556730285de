"""Pins for the oracle's virtual head attention (cross-head low-rank mix with
an identity skip, applied to the gated output of each position).

What pins it, none of which retypes its formula: one-hot factors, whose
effect is a named head receiving another named head's row (this fixes which
factor reads and which writes); zero factors (the identity); a complementary
projector built by QR, which must be idempotent and annihilate its subspace;
and, through the attention oracles, the position of the gate (a head whose
gate is closed still receives the mixed-in row).  Planted mistakes check that
these pins fail when the mix is transposed, loses its identity skip, or runs
before the gate."""
import numpy as np
import pytest

import oracle.hca_oracle as O

RNG = np.random.default_rng(21)


def _x(n=3, H=8, D=5):
    return RNG.standard_normal((n, H, D))


def pin_error(mix=O.vha_mix, prefill=O.prefill_forward, decode=O.decode_forward):
    """Number of violated pins (0 when all hold)."""
    bad = 0
    H, D = 8, 5
    x = _x(4, H, D)
    # one-hot factors: head a receives head b's row, nothing else changes
    a, b = 2, 5
    down = np.zeros((H, 1)); down[b, 0] = 1.0
    up = np.zeros((H, 1)); up[a, 0] = 1.0
    y = mix(x, down, up)
    want = x.copy(); want[:, a] += x[:, b]
    bad += int(not np.allclose(y, want, rtol=0, atol=1e-15))
    # zero factors: the identity, exactly
    r = 3
    bad += int(not np.array_equal(mix(x, np.zeros((H, r)), RNG.standard_normal((H, r))), x))
    # complementary projector I - Q Q^T (Q orthonormal, rank 3): idempotent and
    # annihilates span(Q)
    Q, _ = np.linalg.qr(RNG.standard_normal((H, 3)))
    y1 = mix(x, Q, -Q)
    bad += int(not np.allclose(mix(y1, Q, -Q), y1, atol=1e-12))
    bad += int(not np.allclose(np.einsum("hr,nhd->nrd", Q, y1), 0.0, atol=1e-12))
    # gate position, through the attention oracles: head a's gate closed
    # (sigmoid(-60) ~ 1e-26), head b's open; with the one-hot mix head a's output
    # is head b's gated output, which a mix before the gate would zero
    B, T, Hh, Dd = 1, 40, 4, 8
    q = RNG.standard_normal((B, T, Hh, Dd))
    k = RNG.standard_normal((B, T, Dd))
    v = RNG.standard_normal((B, T, Dd))
    s = RNG.standard_normal((B, T))
    g = RNG.standard_normal((B, T, Hh, Dd))
    g[:, :, 1] = -60.0
    g[:, :, 3] = 60.0
    dn = np.zeros((Hh, 1)); dn[3, 0] = 1.0
    upv = np.zeros((Hh, 1)); upv[1, 0] = 1.0
    out = prefill(q, k, v, s, g, blk=8, win=8, vha=(dn, upv))
    bad += int(not np.allclose(out[:, :, 1], out[:, :, 3], rtol=0, atol=1e-12))
    bad += int(np.abs(out[:, :, 3]).max() < 1e-3)
    # decode agrees with the last position of prefill under the same mix
    dn2 = RNG.standard_normal((Hh, 2)) * 0.3
    up2 = RNG.standard_normal((Hh, 2)) * 0.3
    full = prefill(q, k, v, s, g, blk=8, win=8, vha=(dn2, up2))
    ck, cv = O.compress(k, v, s, 8)
    t = T - 1
    wk = np.zeros((1, 8, Dd)); wv = np.zeros((1, 8, Dd))
    for p_ in range(t - 7, t + 1):
        wk[0, p_ % 8] = k[0, p_]
        wv[0, p_ % 8] = v[0, p_]
    dec = decode(q[:, t], ck, cv, wk, wv, [T], g[:, t], blk=8, win=8, vha=(dn2, up2))
    bad += int(not np.allclose(dec[0], full[0, t], atol=1e-12))
    return bad


def test_vha_pins():
    assert pin_error() == 0


def _transposed(x, down, up):
    return O.vha_mix(x, up, down)


def _no_identity(x, down, up):
    return O.vha_mix(x, down, up) - np.asarray(x, dtype=np.float64)


def _mix_before_gate_prefill(q, k, v, s, g, vha=None, **kw):
    """Planted: the mix runs on the ungated output, then the gate."""
    o = O.prefill_forward(q, k, v, np.asarray(s), np.full_like(g, 60.0), **kw)
    return O.sigmoid(np.asarray(g, dtype=np.float64)) * O.vha_mix(o, *vha)


@pytest.mark.parametrize("kw", [{"mix": _transposed}, {"mix": _no_identity},
                                {"prefill": _mix_before_gate_prefill}],
                         ids=["transposed", "no_identity", "mix_before_gate"])
def test_vha_pins_catch_planted_mistakes(kw):
    try:
        bad = pin_error(**kw)
    except Exception:   # a crash also counts as caught
        bad = 1
    assert bad > 0
