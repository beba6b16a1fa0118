"""Parity of the CUDA decode step (muir_recurrent_step) against the fp64 oracle.

Both sides read the same seeded inputs (gated_delta_rule_115_b200.inputs); the
oracle upcasts the exact bf16/fp32 values to float64.  Error metric: max
absolute error over a tensor divided by the max absolute reference value
(normwise max).  Tolerances: 2e-3 for bf16 inputs and 1e-5 for fp32 inputs on
o and S.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else a
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


@pytest.fixture(scope="module")
def muir():
    import gated_delta_rule_115_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("gmode", ["dynamic", "static", "none"])
def test_decode_parity_small(muir, oracle_mod, D, dtype, gmode):
    from gated_delta_rule_115_b200 import inputs as I
    B, H, steps = 3, 2, 24
    S0, gstat = I.decode_state(B=B, H=H, dk=D, dv=D, seed=77)
    S = S0.cuda()
    Sr = S0.double().numpy()
    for t in range(steps):
        tok = I.decode_tokens(t, B=B, H=H, dk=D, dv=D, seed=77, dtype="bf16" if dtype == torch.bfloat16 else "fp32")
        if gmode == "dynamic":
            gam = torch.sigmoid(torch.randn(B, H, D, generator=torch.Generator().manual_seed(t))).to(dtype)
        elif gmode == "static":
            gam = gstat.to(dtype)
        else:
            gam = None
        dev = {k: v.cuda() for k, v in tok.items()}
        o = muir.recurrent_step(dev["q"], dev["k"], dev["v"], dev["g"], dev["e"], dev["w"],
                                None if gam is None else gam.cuda(), S,
                                gamma_static=(gmode == "static"), out_dtype=torch.float32)
        ro, Sr = oracle_mod.step(tok["q"], tok["k"], tok["v"], tok["g"], tok["e"], tok["w"],
                                 gam, Sr, gamma_static=(gmode == "static"))
        torch.cuda.synchronize()
        assert nmax(o, ro) < TOL[dtype], (t, nmax(o, ro))
    assert nmax(S, Sr) < TOL[dtype]


def test_decode_bf16_output(muir):
    from gated_delta_rule_115_b200 import inputs as I
    S0, gstat = I.decode_state(B=4, H=4)
    tok = {k: v.cuda() for k, v in I.decode_tokens(0, B=4, H=4).items()}
    S1, S2 = S0.cuda(), S0.cuda()
    a = muir.recurrent_step(*[tok[n] for n in "qkvgew"], gstat.cuda(), S1, gamma_static=True,
                            out_dtype=torch.float32)
    b = muir.recurrent_step(*[tok[n] for n in "qkvgew"], gstat.cuda(), S2, gamma_static=True,
                            out_dtype=torch.bfloat16)
    assert b.dtype == torch.bfloat16
    assert torch.equal(a.to(torch.bfloat16), b)
    assert torch.equal(S1, S2)


def test_decode_10k_steps_full_size(muir, oracle_mod):
    """The streaming-decode workload at full size: B=64, H=16, d=128, bf16
    tokens, fp32 state S0 ~ N(0,1), static gamma, 10,000 consecutive steps on
    the GPU; o and S of sampled heads compared with the oracle every 1,000
    steps (heads are independent, so a sampled head is checked exactly)."""
    from gated_delta_rule_115_b200 import inputs as I
    W = I.WORKLOADS[4]
    S0, gstat = I.decode_state()
    S = S0.cuda()
    rng = np.random.default_rng(4)
    sb = np.sort(rng.choice(W.B, 4, replace=False))
    sh = np.sort(rng.choice(W.H, 3, replace=False))
    Sr = S0.double().numpy()[sb][:, sh]
    g_s = gstat[sh]
    worst_o = worst_S = 0.0
    for t in range(W.steps):
        tok = I.decode_tokens(t)
        dev = {k: v.cuda(non_blocking=True) for k, v in tok.items()}
        o = muir.recurrent_step(dev["q"], dev["k"], dev["v"], dev["g"], dev["e"], dev["w"],
                                gstat.cuda(), S, gamma_static=True, out_dtype=torch.float32)
        sub = {k: v[sb][:, sh] for k, v in tok.items()}
        ro, Sr = oracle_mod.step(sub["q"], sub["k"], sub["v"], sub["g"], sub["e"], sub["w"],
                                 g_s, Sr, gamma_static=True)
        if (t + 1) % 1000 == 0:
            torch.cuda.synchronize()
            eo = nmax(o.cpu()[sb][:, sh], ro)
            eS = nmax(S.cpu()[sb][:, sh], Sr)
            worst_o, worst_S = max(worst_o, eo), max(worst_S, eS)
            assert eo < 2e-3 and eS < 2e-3, (t + 1, eo, eS)
    print(f"decode 10k steps: worst o err {worst_o:.2e}, worst S err {worst_S:.2e}")
