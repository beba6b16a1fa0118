"""Pins of the fp64 oracle of the q/k feature prologue, y = SiLU(x) / ||SiLU(x)||
per row ("Muir", wolonglab.org page, "Methodology" and fig. 3(b)), and of its
gradient.  Each pin is fixed by something other than the oracle's own formula:
closed forms of SiLU on special rows, the unit-norm invariant, the zero row,
and central finite differences of the forward for the gradient.
"""
import math

import numpy as np
import pytest


@pytest.fixture(scope="module")
def orc():
    import oracle
    return oracle


def test_unit_norm(orc):
    rng = np.random.default_rng(1)
    x = rng.normal(size=(50, 128)) * rng.uniform(0.1, 5.0, size=(50, 1))
    y = orc.qk_prologue(x)
    assert np.abs(np.linalg.norm(y, axis=-1) - 1.0).max() < 1e-14


def test_zero_row_maps_to_zero(orc):
    y = orc.qk_prologue(np.zeros((3, 64)))
    assert np.all(y == 0.0)


def test_single_channel_row_is_its_sign(orc):
    """One nonzero channel a: SiLU(a) has the sign of a, so y is +-1 there."""
    for a, sign in [(0.3, 1.0), (-2.0, -1.0), (7.0, 1.0)]:
        x = np.zeros(64)
        x[17] = a
        y = orc.qk_prologue(x[None])[0]
        assert y[17] == pytest.approx(sign, abs=1e-15)
        assert np.count_nonzero(y) == 1


def test_antisymmetric_pair_ratio(orc):
    """Row (a, -a): SiLU(a) / SiLU(-a) = -sig(a)/sig(-a) = -e^a, so
    y = (e^a, -1) / sqrt(e^(2a) + 1).  A wrong sign inside the sigmoid, or a
    plain sigmoid instead of SiLU, breaks this."""
    for a in [0.25, 1.0, 3.0]:
        y = orc.qk_prologue(np.array([[a, -a]]))[0]
        den = math.sqrt(math.exp(2 * a) + 1.0)
        assert y[0] == pytest.approx(math.exp(a) / den, rel=1e-13)
        assert y[1] == pytest.approx(-1.0 / den, rel=1e-13)


def test_large_positive_row_is_plain_normalisation(orc):
    """For x >> 0, SiLU(x) = x up to e^-x, so y = x / ||x||: (30, 40) -> (0.6, 0.8)."""
    y = orc.qk_prologue(np.array([[30.0, 40.0]]))[0]
    assert np.abs(y - np.array([0.6, 0.8])).max() < 1e-12


def _fd_grad(orc, x, c, h=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        g[idx] = ((orc.qk_prologue(xp) * c).sum() - (orc.qk_prologue(xm) * c).sum()) / (2 * h)
    return g


def test_gradient_matches_finite_differences(orc):
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 8))
    x[1] *= 4.0
    c = rng.normal(size=(3, 8))
    g = orc.qk_prologue_bwd(x, c)
    assert np.abs(g - _fd_grad(orc, x, c)).max() < 1e-8


def test_gradient_of_constant_norm_is_zero(orc):
    """||y||^2 = 1 whatever x is, so with dy = 2y the gradient vanishes."""
    rng = np.random.default_rng(3)
    x = rng.normal(size=(10, 64))
    y = orc.qk_prologue(x)
    assert np.abs(orc.qk_prologue_bwd(x, 2.0 * y)).max() < 1e-13


def test_gradient_of_zero_row(orc):
    """Below the guard y = s / eps, so dx = dy * SiLU'(0) / eps = dy / (2 eps)."""
    dy = np.linspace(-1.0, 1.0, 64)[None] * 1e-12
    g = orc.qk_prologue_bwd(np.zeros((1, 64)), dy)
    assert np.abs(g - dy / (2.0 * orc.QK_NORM_EPS)).max() < 1e-15
