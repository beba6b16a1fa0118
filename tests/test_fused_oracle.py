"""Pins of the fp64 oracle's output gate (o * sigmoid(z)) and of the fused layer
(q/k prologue -> recurrence -> output gate, "Muir", wolonglab.org page,
"Methodology" and fig. 3(b)).  Each is fixed by something other than the
oracle's own formula: closed values of the sigmoid, its limits, and central
finite differences of the forward for every gradient of the composed chain.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.fixture(scope="module")
def orc():
    import oracle
    return oracle


def test_gate_closed_values(orc):
    rng = np.random.default_rng(3)
    o = rng.normal(size=(2, 3, 2, 5))
    # sigmoid(0) = 1/2 exactly, sigmoid(ln 3) = 3/4
    assert np.array_equal(orc.out_gate(o, np.zeros_like(o)), o / 2)
    assert np.abs(orc.out_gate(o, np.full_like(o, math.log(3.0))) - 0.75 * o).max() < 1e-15
    # open gate: sigmoid(40) = 1 - 4e-18 -> o; closed gate: sigmoid(-40) ~ 4e-18 -> 0
    assert np.abs(orc.out_gate(o, np.full_like(o, 40.0)) - o).max() < 1e-15
    assert np.abs(orc.out_gate(o, np.full_like(o, -40.0))).max() < 1e-16


def test_gate_gradient_at_zero(orc):
    """At z = 0: d/do = 1/2 and d/dz = o sig'(0) = o / 4."""
    rng = np.random.default_rng(4)
    o, dy = rng.normal(size=(7, 3)), rng.normal(size=(7, 3))
    do, dz = orc.out_gate_bwd(o, np.zeros_like(o), dy)
    assert np.array_equal(do, dy / 2)
    assert np.abs(dz - dy * o / 4).max() < 1e-16


def test_gate_gradient_finite_differences(orc):
    rng = np.random.default_rng(5)
    o, z, dy = (rng.normal(size=(4, 6)) for _ in range(3))
    do, dz = orc.out_gate_bwd(o, z, dy)
    h = 1e-6
    f = lambda oo, zz: float((dy * orc.out_gate(oo, zz)).sum())
    for idx in np.ndindex(*o.shape):
        e = np.zeros_like(o)
        e[idx] = h
        assert (f(o + e, z) - f(o - e, z)) / (2 * h) == pytest.approx(do[idx], abs=1e-8)
        assert (f(o, z + e) - f(o, z - e)) / (2 * h) == pytest.approx(dz[idx], abs=1e-8)


def test_fused_prologue_on_large_rows_is_plain_normalisation(orc):
    """Raw rows with every entry >= 30: SiLU(x) = x up to e^-30, so the fused
    forward with raw q and k equals the plain forward on x / ||x||."""
    rng = np.random.default_rng(6)
    B, T, H, d = 1, 9, 2, 4
    xq, xk = (30 + 10 * rng.random(size=(B, T, H, d)) for _ in range(2))
    v = rng.normal(size=(B, T, H, d))
    g = -rng.random(size=(B, T, H, d))
    e, w, ga = (rng.random(size=(B, T, H, d)) for _ in range(3))
    nq = xq / np.linalg.norm(xq, axis=-1, keepdims=True)
    nk = xk / np.linalg.norm(xk, axis=-1, keepdims=True)
    og, S, o = orc.fwd_fused(xq, xk, v, g, e, w, ga, qk_raw=True)
    r_o, r_S = orc.fwd(nq, nk, v, g, e, w, ga)
    assert np.abs(o - r_o).max() < 1e-11 and np.abs(S - r_S).max() < 1e-11
    assert np.array_equal(og, o)


def test_fused_gradients_finite_differences(orc):
    """Every gradient of bwd_fused (raw q, k, the gates, v, S0 and the output
    gate's z) against central differences of fwd_fused's loss
    sum(o_gated * dO) + sum(S_T * dS)."""
    rng = np.random.default_rng(7)
    B, T, H, d = 1, 5, 1, 3
    x = dict(q=rng.normal(size=(B, T, H, d)), k=rng.normal(size=(B, T, H, d)),
             v=rng.normal(size=(B, T, H, d)), g=-rng.random(size=(B, T, H, d)),
             e=rng.random(size=(B, T, H, d)), w=rng.random(size=(B, T, H, d)),
             gamma=rng.random(size=(B, T, H, d)), S0=rng.normal(size=(B, H, d, d)),
             z_out=rng.normal(size=(B, T, H, d)))
    dO, dS = rng.normal(size=(B, T, H, d)), rng.normal(size=(B, H, d, d))

    def loss(y):
        og, S, _ = orc.fwd_fused(y["q"], y["k"], y["v"], y["g"], y["e"], y["w"], y["gamma"],
                                 y["S0"], z_out=y["z_out"], qk_raw=True)
        return float((og * dO).sum() + (S * dS).sum())

    gr = orc.bwd_fused(x["q"], x["k"], x["v"], x["g"], x["e"], x["w"], x["gamma"], x["S0"],
                       dO=dO, dS_final=dS, z_out=x["z_out"], qk_raw=True)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "e": "de", "w": "dw",
             "gamma": "dgamma", "S0": "dS0", "z_out": "dz_out"}
    h = 1e-6
    for n, gn in names.items():
        for idx in np.ndindex(*x[n].shape):
            yp = {m: a.copy() for m, a in x.items()}
            ym = {m: a.copy() for m, a in x.items()}
            yp[n][idx] += h
            ym[n][idx] -= h
            fd = (loss(yp) - loss(ym)) / (2 * h)
            assert fd == pytest.approx(gr[gn][idx], abs=2e-7, rel=1e-6), (n, idx)
