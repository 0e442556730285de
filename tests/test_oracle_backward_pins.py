"""Pins for the oracle's backward pass: central finite differences of the
forward oracle (itself pinned by brute force and library routines) along
random directions and single coordinates of every input, on small problems
(blk = win = 4 or 8) that span several compressed blocks, a ragged tail and
positions whose window reaches back past block boundaries.  Planted mistakes
(the oracle with one line of its arithmetic replaced: a dropped
softmax-Jacobian term, swapped key/value gradients, a compressor weight
dropped, uncentred score gradients, a gate derivative without its
(1 - sigmoid) factor) must fail them."""
import inspect
import textwrap

import numpy as np
import pytest

import oracle.hca_oracle as O

EPS = 1e-5


def _problem(seed, B=1, T=23, H=2, D=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, D))
    v = rng.standard_normal((B, T, D))
    s = rng.standard_normal((B, T)) * 1.5
    g = rng.standard_normal((B, T, H, D))
    dout = rng.standard_normal((B, T, H, D))
    return [q, k, v, s, g], dout


def _loss(x, dout, blk, win):
    return float((O.prefill_forward(*x, blk=blk, win=win) * dout).sum())


def pin_error(backward=O.prefill_backward, blk=4, win=4, seed=0, B=1, T=23):
    """Largest relative disagreement between the analytic gradients and
    central differences (directional, plus a few coordinates)."""
    x, dout = _problem(seed, B=B, T=T)
    grads = backward(*x, dout, blk=blk, win=win)
    rng = np.random.default_rng(seed + 100)
    worst = 0.0
    for i, gr in enumerate(grads):
        for trial in range(3):
            u = rng.standard_normal(x[i].shape)
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[i] = x[i] + EPS * u
            xm[i] = x[i] - EPS * u
            fd = (_loss(xp, dout, blk, win) - _loss(xm, dout, blk, win)) / (2 * EPS)
            an = float((gr * u).sum())
            worst = max(worst, abs(fd - an) / max(1e-6, abs(fd)))
        flat = np.argsort(np.abs(gr).ravel())[-2:]    # the two largest entries
        for f in flat:
            e = np.zeros(x[i].size)
            e[f] = 1.0
            e = e.reshape(x[i].shape)
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[i] = x[i] + EPS * e
            xm[i] = x[i] - EPS * e
            fd = (_loss(xp, dout, blk, win) - _loss(xm, dout, blk, win)) / (2 * EPS)
            worst = max(worst, abs(fd - gr.ravel()[f]) / max(1e-6, abs(fd)))
    return worst


@pytest.mark.parametrize("blk,win,seed,B,T", [(4, 4, 0, 1, 23), (8, 8, 1, 2, 37),
                                              (4, 8, 2, 1, 30), (8, 4, 3, 1, 26)])
def test_backward_matches_finite_differences(blk, win, seed, B, T):
    assert pin_error(blk=blk, win=win, seed=seed, B=B, T=T) < 1e-6


def test_backward_gate_closed_form():
    """dg = dout * o * sigmoid'(g), o the ungated output (forward at g = +60)."""
    x, dout = _problem(5)
    q, k, v, s, g = x
    o = O.prefill_forward(q, k, v, s, np.full_like(g, 60.0), blk=4, win=4)
    sg = O.sigmoid(g)
    *_, dg = O.prefill_backward(q, k, v, s, g, dout, blk=4, win=4)
    assert np.allclose(dg, dout * o * sg * (1 - sg), rtol=1e-12, atol=1e-14)


def _mutant(old: str, new: str):
    """The oracle's backward with one line of its arithmetic replaced."""
    src = textwrap.dedent(inspect.getsource(O.prefill_backward))
    assert src.count(old) == 1, old
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["prefill_backward"]


MUTANTS = {
    "no_jacobian_term": ("dz = P * (dP - (P * dP).sum(axis=-1, keepdims=True))", "dz = P * dP"),
    "keys_values_swapped": ('dvals = np.einsum("nhk,nhd->kd", P, dO)',
                            'dvals = np.einsum("nhk,nhd->kd", dz, qr)'),
    "compressor_weight_dropped": ("dk[b, sl] += w[:, None] * dck[b, j]", "dk[b, sl] += dck[b, j]"),
    "score_grad_no_centering": ("ds[b, sl] = w * (a - (w * a).sum())", "ds[b, sl] = w * a"),
    "gate_factor": ("dg[b, t_lo : t_hi + 1] = do * o * sg * (1.0 - sg)",
                    "dg[b, t_lo : t_hi + 1] = do * o * sg"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_pins_catch_planted_mistakes(name):
    assert pin_error(backward=_mutant(*MUTANTS[name])) > 1e-3
