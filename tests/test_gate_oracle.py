"""Pins of the fp64 oracle of the fused low-rank gate projection ("Muir",
wolonglab.org page, "Methodology", eq:ours_proj; fig. 3(c): one latent per
token, five up-projections of ranks (64, 64, 128, 128, 128), channel biases).
Each pin is fixed by something other than the oracle's formula: closed values
of the activations, a brute-force loop for the up-projection, one-hot latents
for the column layout, torch's own bf16 conversion for the rounding, and
central finite differences for the gradient.
"""
import math

import numpy as np
import pytest
import torch


@pytest.fixture(scope="module")
def orc():
    import oracle
    return oracle


def make(rng, B=1, T=3, H=2, d=4, ranks=(2, 2, 3, 3, 3), scale=1.0):
    offs, ups, o = {}, {}, 0
    for fam, r in zip(("f", "b", "g", "w", "q"), ranks):
        ups[fam] = (o, rng.normal(size=(r, H * d)) * scale, rng.normal(size=H * d) * scale)
        o += r
    lat = rng.normal(size=(B, T, o))
    return lat, ups


def test_zero_latent_closed_values(orc):
    rng = np.random.default_rng(0)
    lat, ups = make(rng)
    lat[:] = 0.0
    ups = {f: (o, U, np.zeros_like(b)) for f, (o, U, b) in ups.items()}
    gt = orc.gate_projection(lat, ups, H=2, rounded=False)
    assert np.abs(gt["g"] + math.log(2.0)).max() < 1e-15      # -softplus(0) = -ln 2
    for n in ("e", "w", "gamma"):
        assert np.array_equal(gt[n], np.full_like(gt[n], 0.5))  # sigmoid(0) = 1/2
    assert np.array_equal(gt["z_out"], np.zeros_like(gt["z_out"]))
    # biases alone: sigmoid(ln 3) = 3/4, -softplus(ln(e - 1)) = -1
    ups2 = {f: (o, U, np.full_like(b, math.log(math.e - 1) if f == "f" else math.log(3.0)))
            for f, (o, U, b) in ups.items()}
    gt2 = orc.gate_projection(lat, ups2, H=2, rounded=False)
    assert np.abs(gt2["g"] + 1.0).max() < 1e-15
    assert np.abs(gt2["e"] - 0.75).max() < 1e-15
    assert np.abs(gt2["z_out"] - math.log(3.0)).max() < 1e-15


def test_up_projection_brute_force(orc):
    rng = np.random.default_rng(1)
    H, d = 2, 4
    lat, ups = make(rng, B=2, T=3, H=H, d=d)
    pre = orc.gate_pre(lat, ups, H)
    for fam, (off, U, bias) in ups.items():
        r = U.shape[0]
        for b in range(2):
            for t in range(3):
                for h in range(H):
                    for c in range(d):
                        s = bias[h * d + c]
                        for i in range(r):
                            s += lat[b, t, off + i] * U[i, h * d + c]
                        assert pre[fam][b, t, h, c] == pytest.approx(s, abs=1e-13)


def test_latent_layout_one_hot(orc):
    """A latent that is 1 in one column selects that row of its family's U
    (plus the bias) and leaves every other family at its bias."""
    rng = np.random.default_rng(2)
    H, d = 2, 4
    lat, ups = make(rng, H=H, d=d)
    for fam, (off, U, bias) in ups.items():
        for i in range(U.shape[0]):
            z = np.zeros_like(lat)
            z[:, :, off + i] = 1.0
            pre = orc.gate_pre(z, ups, H)
            for f2, (o2, U2, b2) in ups.items():
                want = (U2[i] if f2 == fam else 0.0) + b2
                assert np.abs(pre[f2].reshape(*z.shape[:2], -1) - want).max() < 1e-15


def test_round_bf16_matches_torch(orc):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.integers(-6, 6, size=4000),
                        [1.00390625, 1.01171875, -2.0 ** -130, 0.0, -0.0]])
    want = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.round_bf16(x), want)


def test_gradients_finite_differences(orc):
    rng = np.random.default_rng(4)
    H, d = 2, 3
    lat, ups = make(rng, B=1, T=2, H=H, d=d, ranks=(2, 2, 2, 2, 2), scale=0.7)
    dg = {n: rng.normal(size=(1, 2, H, d)) for n in ("g", "e", "z_out", "w", "gamma")}

    def loss(lat_, ups_):
        gt = orc.gate_projection(lat_, ups_, H, rounded=False)
        return float(sum((dg[n] * gt[n]).sum() for n in dg))

    res = orc.gate_projection_bwd(lat, ups, H, dg)
    h = 1e-6
    for idx in np.ndindex(*lat.shape):
        e = np.zeros_like(lat)
        e[idx] = h
        fd = (loss(lat + e, ups) - loss(lat - e, ups)) / (2 * h)
        assert fd == pytest.approx(res["dlat"][idx], abs=1e-7)
    for fam, (off, U, bias) in ups.items():
        for idx in np.ndindex(*U.shape):
            e = np.zeros_like(U)
            e[idx] = h
            up = dict(ups); um = dict(ups)
            up[fam] = (off, U + e, bias); um[fam] = (off, U - e, bias)
            fd = (loss(lat, up) - loss(lat, um)) / (2 * h)
            assert fd == pytest.approx(res["dU_" + fam][idx], abs=1e-7)
        for j in range(bias.size):
            e = np.zeros_like(bias)
            e[j] = h
            up = dict(ups); um = dict(ups)
            up[fam] = (off, U, bias + e); um[fam] = (off, U, bias - e)
            fd = (loss(lat, up) - loss(lat, um)) / (2 * h)
            assert fd == pytest.approx(res["dbias_" + fam][j], abs=1e-7)
