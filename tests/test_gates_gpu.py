"""Parity of the fused low-rank gate projection (muir_chunk_fwd_fused /
muir_chunk_bwd_fused with a latent; "Muir", wolonglab.org page,
"Methodology", eq:ours_proj, fig. 3(c)) against the fp64 oracle: the gates
``oracle.gate_projection`` forms from the same latent, up-projections and
biases (bf16-rounded, the gate dtype the kernels consume), fed to the oracle's
fused layer, and the gradients through ``oracle.gate_projection_bwd``.

Metric: max |gpu - oracle| / max |oracle| per tensor; 2e-3 on o and the final
state, 5e-3 on the per-token gradients (dq, dk, dv, dlatent, the gates' own), as
elsewhere.  The kernels form each pre-activation in float32 on the tensor cores
before the bf16 rounding that the oracle takes from its float32 rounding, so a
handful of gate values can sit one bf16 unit apart; the bounds include that.

dU and dbias are sums over every token of per-token terms, each carrying the
per-token gradient allowance; where the sum cancels, the relative error of the
total exceeds that of its terms.  Their bound is therefore derived from the
per-token one: |d dbias[c]| <= sum_t |act'(pre)[t][c]| * 5e-3 max|dgate| and
|d dU[i][c]| <= sum_t |a[t][i]| |act'(pre)[t][c]| * 5e-3 max|dgate|, taken
relative to max |reference|, never below 5e-3 and at most 2e-2 (the worst-case
alignment of the per-token errors that the derivation assumes is far from what
happens; the cap keeps the check tight).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
FAMILY_GATE = {"f": "g", "b": "e", "g": "z_out", "w": "w", "q": "gamma"}


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


@pytest.fixture(scope="module")
def muir():
    import gated_delta_rule_115_b200 as m
    m.lib()
    return m


@pytest.fixture(autouse=True)
def no_expired_waits(muir):
    muir.device_wait_status()
    yield
    muir.device_wait_status()


@pytest.mark.parametrize("families,raw", [(("f", "b", "g", "w", "q"), False),
                                          (("b", "w"), False),
                                          (("f", "b", "g", "w", "q"), True)])
def test_gate_projection_parity(muir, oracle_mod, families, raw):
    from gated_delta_rule_115_b200 import inputs as I
    B, T, H = 1, 512, 2
    x = I.fused_inputs(2, B=B, T=T, H=H, s0_std=1.0, with_dO=True)
    lat, proj = I.gate_latent_inputs(B, T, H, families=families)
    ups = {f: (off, U.double().numpy(), b.double().numpy()) for f, (off, U, b) in proj.items()}
    gates = oracle_mod.gate_projection(lat.double().numpy(), ups, H)
    # oracle inputs: projected gates replace the tensors of their families
    args = {n: x[n] for n in NAMES}
    if raw:
        args["q"], args["k"] = x["xq"], x["xk"]
    for f in families:
        if f != "g":
            args[FAMILY_GATE[f]] = torch.from_numpy(gates[FAMILY_GATE[f]])
    z = torch.from_numpy(gates["z_out"]) if "g" in families else None
    og, S, o_pre = oracle_mod.fwd_fused(*[args[n] for n in NAMES], S0=x["S0"], z_out=z, qk_raw=raw)
    gr = oracle_mod.bwd_fused(*[args[n] for n in NAMES], S0=x["S0"], dO=x["dO"], z_out=z, qk_raw=raw)
    dgates = {FAMILY_GATE[f]: gr["dz_out" if f == "g" else "d" + FAMILY_GATE[f]] for f in families}
    pg = oracle_mod.gate_projection_bwd(lat.double().numpy(), ups, H, dgates)

    # GPU: gate tensors of projected families are not passed
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    din = {n: d[n] for n in NAMES}
    if raw:
        din["q"], din["k"] = d["xq"], d["xk"]
    for f in families:
        if f != "g":
            din[FAMILY_GATE[f]] = None
    latd = lat.cuda()
    projd = {f: (off, U.cuda(), b.cuda()) for f, (off, U, b) in proj.items()}
    o, Sf, sv = muir.chunk_fwd_fused(*[din[n] for n in NAMES], d["S0"], qk_raw=raw,
                                     out_dtype=torch.float32, latent=latd, proj=projd)
    g = muir.chunk_bwd_fused(*[din[n] for n in NAMES], d["S0"], d["dO"], qk_raw=raw, saved=sv,
                             latent=latd, proj=projd)
    torch.cuda.synchronize()
    # bounds of the token sums (dU, dbias), from the per-token allowance
    latn = lat.double().numpy().reshape(B * T, -1)
    pre = oracle_mod.gate_pre(latn.reshape(B, T, -1), ups, H)
    bound = {}
    for f in families:
        p_ = pre[f].reshape(B * T, -1)
        sg = 1.0 / (1.0 + np.exp(-p_))
        ag = np.abs(-sg if f == "f" else (np.ones_like(p_) if f == "g" else sg * (1.0 - sg)))
        allow = 5e-3 * np.abs(dgates[FAMILY_GATE[f]]).max()
        off, Uf, _ = ups[f]
        a_ = np.abs(latn[:, off:off + Uf.shape[0]])
        bound["dbias_" + f] = min(2e-2, max(5e-3, allow * ag.sum(0).max() / np.abs(pg["dbias_" + f]).max()))
        bound["dU_" + f] = min(2e-2, max(5e-3, allow * (a_.T @ ag).max() / np.abs(pg["dU_" + f]).max()))
    errs = {"o": nmax(o, og), "S": nmax(Sf, S), "dq": nmax(g["dq"], gr["dq"]),
            "dk": nmax(g["dk"], gr["dk"]), "dv": nmax(g["dv"], gr["dv"]),
            "dS0": nmax(g["dS0"], gr["dS0"]), "dlatent": nmax(g["dlatent"], pg["dlat"])}
    for f in families:
        errs["dU_" + f] = nmax(g["dU_" + f], pg["dU_" + f])
        errs["dbias_" + f] = nmax(g["dbias_" + f], pg["dbias_" + f])
    for n, gn in (("e", "de"), ("w", "dw"), ("gamma", "dgamma"), ("g", "dg")):
        if gn in g:
            errs[gn] = nmax(g[gn], gr[gn])
    print(f"gates {families} raw={raw}: " + " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    print("  sum bounds: " + " ".join(f"{n} {v:.2e}" for n, v in bound.items()))
    assert errs["o"] < 2e-3 and errs["S"] < 2e-3, errs
    for n, v in errs.items():
        if n not in ("o", "S"):
            assert v < bound.get(n, 5e-3), (n, v, bound.get(n, 5e-3))
