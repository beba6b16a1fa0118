"""Pins of the fp64 oracle against facts that do not come from the oracle.

The recurrence (wolonglab.org page on arXiv 2611.08376, "Methodology",
eq:gdn2 / eq:ours), per head with state S (rows = key channels):

    S_t = D_t S_{t-1} - (e_t*k_t)(k_t^T D_t S_{t-1}) + k_t (w_t*v_t)^T,
    o_t = S_t^T (gamma_t*q_t),   D_t = diag(exp g_t).

Each test fixes a part of it through something other than the oracle's own
code: a closed form of a special case (linear attention, gated linear
attention, the delta rule, pure decay), an invariant that follows from the
algebra (exact retrieval), a hand-worked example, structural properties
(linearity, channel equivariance, state passing, chunk-size invariance between
two independent C sources), and for the gradients central finite differences
and torch autograd.  Shapes use d_k != d_v so that a transposed operand fails.
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_inputs(seed, B=1, T=24, H=2, dk=5, dv=3, unit_k=True, s0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    e = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
    w = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))
    gm = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    return dict(q=q, k=k, v=v, g=g, e=e, w=w, gamma=gm, S0=S0)


def rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ------------------------------------------------------------ closed forms

def test_hand_worked_example(oracle_mod):
    """Two tokens computed by hand (tests/golden/hand_example_T2_d2.json)."""
    with open(os.path.join(HERE, "golden", "hand_example_T2_d2.json")) as f:
        fx = json.load(f)
    x = {k: np.array(v) for k, v in fx["inputs"].items()}
    o, S = oracle_mod.fwd(**x)
    tol = fx["tolerance_abs"]
    assert np.abs(o - np.array(fx["expected"]["o"])).max() < tol
    assert np.abs(S - np.array(fx["expected"]["S_final"])).max() < tol
    oc, Sc, _ = oracle_mod.chunk_fwd(**x, chunk=2)
    assert np.abs(oc - np.array(fx["expected"]["o"])).max() < tol
    assert np.abs(Sc - np.array(fx["expected"]["S_final"])).max() < tol


def test_linear_attention_closed_form(oracle_mod):
    """e = 0, g = 0: o_t = S0^T qh_t + sum_{s<=t} (k_s . qh_t) (w_s*v_s)."""
    x = rand_inputs(1, unit_k=False)
    x["e"][:] = 0.0
    x["g"][:] = 0.0
    o, S = oracle_mod.fwd(**x)
    qh = x["gamma"] * x["q"]
    u = x["w"] * x["v"]
    B, T, H, dk = qh.shape
    ref = np.zeros_like(o)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                acc = x["S0"][b, h].T @ qh[b, t, h]
                for s in range(t + 1):
                    acc = acc + (x["k"][b, s, h] @ qh[b, t, h]) * u[b, s, h]
                ref[b, t, h] = acc
    assert rel(o, ref) < 1e-13
    S_ref = x["S0"] + np.einsum("bthj,bthc->bhjc", x["k"], u)
    assert rel(S, S_ref) < 1e-13


def test_gated_linear_attention_closed_form(oracle_mod):
    """e = 0, any g: o_t = S0^T (qh_t e^{G_t}) + sum_{s<=t} ((qh_t e^{G_t - G_s}) . k_s) u_s,
    with G_t the running sum of g from the first token."""
    x = rand_inputs(2, unit_k=False)
    x["e"][:] = 0.0
    o, S = oracle_mod.fwd(**x)
    qh = x["gamma"] * x["q"]
    u = x["w"] * x["v"]
    G = np.cumsum(x["g"], axis=1)
    B, T, H, dk = qh.shape
    ref = np.zeros_like(o)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                acc = x["S0"][b, h].T @ (qh[b, t, h] * np.exp(G[b, t, h]))
                for s in range(t + 1):
                    f = np.exp(G[b, t, h] - G[b, s, h])
                    acc = acc + ((qh[b, t, h] * f) @ x["k"][b, s, h]) * u[b, s, h]
                ref[b, t, h] = acc
    assert rel(o, ref) < 1e-12


def test_delta_rule(oracle_mod):
    """g = 0, e = w = 1: Widrow-Hoff, S_t = S_{t-1} + k_t (v_t - S_{t-1}^T k_t)^T."""
    x = rand_inputs(3)
    x["g"][:] = 0.0
    x["e"][:] = 1.0
    x["w"][:] = 1.0
    o, S = oracle_mod.fwd(**x)
    B, T, H, dk = x["q"].shape
    ref = np.zeros_like(o)
    S_ref = x["S0"].copy()
    for b in range(B):
        for h in range(H):
            St = S_ref[b, h]
            for t in range(T):
                kt = x["k"][b, t, h]
                err = x["v"][b, t, h] - St.T @ kt
                St = St + np.outer(kt, err)
                ref[b, t, h] = St.T @ (x["gamma"][b, t, h] * x["q"][b, t, h])
            S_ref[b, h] = St
    assert rel(o, ref) < 1e-12
    assert rel(S, S_ref) < 1e-12


def test_exact_retrieval_invariant(oracle_mod):
    """e = 1 and |k_t| = 1 give S_t^T k_t = w_t*v_t for any g, w, S0.
    Read it through the oracle's own readout with q = k and gamma = 1."""
    x = rand_inputs(4, T=40)
    x["e"][:] = 1.0
    x["q"] = x["k"].copy()
    x["gamma"][:] = 1.0
    o, _ = oracle_mod.fwd(**x)
    assert np.abs(o - x["w"] * x["v"]).max() < 1e-12


def test_pure_decay(oracle_mod):
    """e = 0, w = 0: S_t = diag(exp(sum g)) S0 and o_t = S_t^T qh_t."""
    x = rand_inputs(5)
    x["e"][:] = 0.0
    x["w"][:] = 0.0
    o, S = oracle_mod.fwd(**x)
    G = np.cumsum(x["g"], axis=1)
    S_ref = np.exp(G[:, -1])[..., None] * x["S0"]
    assert rel(S, S_ref) < 1e-13
    St = np.exp(G)[..., None] * x["S0"][:, None]  # [B,T,H,dk,dv]
    o_ref = np.einsum("bthjc,bthj->bthc", St, x["gamma"] * x["q"])
    assert rel(o, o_ref) < 1e-13


def test_gamma_only_scales_readout(oracle_mod):
    """gamma scales q at readout only: the final state does not depend on it,
    and o is linear in gamma."""
    x = rand_inputs(6)
    o1, S1 = oracle_mod.fwd(**x)
    y = dict(x)
    y["gamma"] = 2.5 * x["gamma"]
    o2, S2 = oracle_mod.fwd(**y)
    assert np.abs(S1 - S2).max() == 0.0
    assert rel(o2, 2.5 * o1) < 1e-14


# ------------------------------------------------------------ invariants

@pytest.mark.parametrize("C", [1, 2, 3, 4, 7, 8, 16, 32, 64])
def test_chunk_size_invariance(oracle_mod, C):
    """The chunked WY oracle (independent C source) equals the token loop for
    every chunk size, including a ragged last chunk (T = 45)."""
    x = rand_inputs(7, T=45, dk=6, dv=4)
    o, S = oracle_mod.fwd(**x)
    oc, Sc, Sch = oracle_mod.chunk_fwd(**x, chunk=C)
    assert rel(oc, o) < 1e-12
    assert rel(Sc, S) < 1e-12
    # chunk-start states equal the token loop's prefix states
    n = Sch.shape[2]
    for i in range(1, n):
        xp = {kk: (vv[:, : i * C] if vv is not None and vv.ndim == 4 else vv) for kk, vv in x.items()}
        _, Sp = oracle_mod.fwd(**xp)
        assert rel(Sch[:, :, i], Sp) < 1e-12


def test_chunk_invariance_strong_decay(oracle_mod):
    """Log decay down to -8 per token (cumulative -512 over a 64 chunk): the
    chunked oracle uses exact exponent differences and still matches."""
    x = rand_inputs(8, T=128, dk=6, dv=4)
    rng = np.random.default_rng(80)
    x["g"] = np.broadcast_to(rng.uniform(-8, -1e-4, (1, 1, 2, 6)), x["g"].shape).copy()
    o, S = oracle_mod.fwd(**x)
    oc, Sc, _ = oracle_mod.chunk_fwd(**x, chunk=64)
    assert rel(oc, o) < 1e-12 and rel(Sc, S) < 1e-12
    assert np.isfinite(oc).all()


def test_linearity_in_v_and_S0(oracle_mod):
    x1 = rand_inputs(9)
    x2 = rand_inputs(10)
    a, b = 0.7, -1.3
    x = dict(x1)
    x["v"] = a * x1["v"] + b * x2["v"]
    x["S0"] = a * x1["S0"] + b * x2["S0"]
    y2 = dict(x1)
    y2["v"], y2["S0"] = x2["v"], x2["S0"]
    o, S = oracle_mod.fwd(**x)
    o1, S1 = oracle_mod.fwd(**x1)
    o2, S2 = oracle_mod.fwd(**y2)
    assert rel(o, a * o1 + b * o2) < 1e-12
    assert rel(S, a * S1 + b * S2) < 1e-12


def test_value_channel_equivariance(oracle_mod):
    x = rand_inputs(11, dv=5)
    perm = np.array([3, 0, 4, 1, 2])
    y = dict(x)
    y["v"] = x["v"][..., perm]
    y["w"] = x["w"][..., perm]
    y["S0"] = x["S0"][..., perm]
    o, S = oracle_mod.fwd(**x)
    op, Sp = oracle_mod.fwd(**y)
    assert rel(op, o[..., perm]) < 1e-14
    assert rel(Sp, S[..., perm]) < 1e-14


def test_state_passing(oracle_mod):
    x = rand_inputs(12, T=30)
    o, S = oracle_mod.fwd(**x)
    first = {k: (v[:, :11] if v is not None and v.ndim == 4 else v) for k, v in x.items()}
    o1, S1 = oracle_mod.fwd(**first)
    second = {k: (v[:, 11:] if v is not None and v.ndim == 4 else v) for k, v in x.items()}
    second["S0"] = S1
    o2, S2 = oracle_mod.fwd(**second)
    assert rel(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert rel(S2, S) < 1e-13


def test_decode_steps_equal_forward(oracle_mod):
    x = rand_inputs(13, T=17, B=2)
    o, S = oracle_mod.fwd(**x)
    St = x["S0"]
    for t in range(17):
        tok = {k: x[k][:, t] for k in ("q", "k", "v", "g", "e", "w", "gamma")}
        ot, St = oracle_mod.step(S=St, **tok)
        assert rel(ot, o[:, t]) < 1e-13
    assert rel(St, S) < 1e-13


def test_decode_static_gamma(oracle_mod):
    x = rand_inputs(14, T=1, B=3, H=2)
    tok = {k: x[k][:, 0] for k in ("q", "k", "v", "g", "e", "w")}
    gs = np.random.default_rng(5).uniform(0.1, 1, (2, 5))
    o1, S1 = oracle_mod.step(gamma=gs, S=x["S0"], gamma_static=True, **tok)
    o2, S2 = oracle_mod.step(gamma=np.broadcast_to(gs, (3, 2, 5)), S=x["S0"], **tok)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_zero_length_and_zero_state(oracle_mod):
    x = rand_inputs(15, T=6, s0=False)
    o, S = oracle_mod.fwd(**x)
    y = dict(x)
    y["S0"] = np.zeros((1, 2, 5, 3))
    o2, S2 = oracle_mod.fwd(**y)
    assert np.array_equal(o, o2) and np.array_equal(S, S2)
    z = {k: (v[:, :0] if v is not None and v.ndim == 4 else v) for k, v in y.items()}
    g = oracle_mod.bwd(**z, dS_final=np.ones((1, 2, 5, 3)))
    assert np.array_equal(g["dS0"], np.ones((1, 2, 5, 3)))


# ------------------------------------------------------------ gradients

GRAD_NAMES = ["q", "k", "v", "g", "e", "w", "gamma", "S0"]


def _loss(oracle_mod, x, dO, dS):
    o, S = oracle_mod.fwd(**x, threads=1)
    return float((o * dO).sum() + (S * dS).sum())


@pytest.mark.parametrize("seed", [21, 22])
def test_bptt_central_differences(oracle_mod, seed):
    x = rand_inputs(seed, T=7, H=1, dk=3, dv=2)
    rng = np.random.default_rng(seed + 100)
    dO = rng.standard_normal((1, 7, 1, 2))
    dS = rng.standard_normal((1, 1, 3, 2))
    gr = oracle_mod.bwd(**x, dO=dO, dS_final=dS, ckpt=3)
    h = 1e-6
    for name in GRAD_NAMES:
        key = "dS0" if name == "S0" else "d" + name
        num = np.zeros_like(x[name])
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = {k: (v.copy() if v is not None else None) for k, v in x.items()}
            xm = {k: (v.copy() if v is not None else None) for k, v in x.items()}
            xp[name][i] += h
            xm[name][i] -= h
            num[i] = (_loss(oracle_mod, xp, dO, dS) - _loss(oracle_mod, xm, dO, dS)) / (2 * h)
        err = np.abs(num - gr[key]).max() / max(np.abs(num).max(), 1e-12)
        assert err < 1e-7, (name, err)


def test_bptt_matches_torch_autograd(oracle_mod):
    """The recurrence restated in torch (float64, CPU), differentiated by
    autograd, against the hand-derived BPTT with several checkpoint sizes."""
    import torch
    x = rand_inputs(31, B=2, T=29, H=2, dk=6, dv=4)
    rng = np.random.default_rng(32)
    dO = rng.standard_normal((2, 29, 2, 4))
    dS = rng.standard_normal((2, 2, 6, 4))
    tx = {k: torch.tensor(v, requires_grad=True) for k, v in x.items()}
    S = tx["S0"]
    outs = []
    for t in range(29):
        D = torch.exp(tx["g"][:, t])[..., None]  # [B,H,dk,1]
        P = D * S
        kt = tx["k"][:, t]
        y = torch.einsum("bhjc,bhj->bhc", P, kt)
        a = tx["e"][:, t] * kt
        u = tx["w"][:, t] * tx["v"][:, t]
        S = P - a[..., None] * y[..., None, :] + kt[..., None] * u[..., None, :]
        outs.append(torch.einsum("bhjc,bhj->bhc", S, tx["gamma"][:, t] * tx["q"][:, t]))
    o = torch.stack(outs, dim=1)
    loss = (o * torch.tensor(dO)).sum() + (S * torch.tensor(dS)).sum()
    loss.backward()
    for ck in (1, 5, 64):
        gr = oracle_mod.bwd(**x, dO=dO, dS_final=dS, ckpt=ck)
        for name in GRAD_NAMES:
            key = "dS0" if name == "S0" else "d" + name
            assert rel(gr[key], tx[name].grad.numpy()) < 1e-12, (name, ck)
