"""Parity of the fused stages (muir_chunk_fwd_fused / muir_chunk_bwd_fused)
against the fp64 oracle's composed layer (``oracle.fwd_fused`` /
``oracle.bwd_fused``): the q/k prologue applied inside the chunk kernels to raw
q and k, and the output gate o * sigmoid(z) in the output epilogue with its
gradient in the backward's first kernel ("Muir", wolonglab.org page,
"Methodology" and fig. 3(b); tab:abl caption).

Metric: max |gpu - oracle| / max |oracle| per tensor.  Bounds: 2e-3 on the
forward outputs and the final state, 5e-3 on gradients (bf16 inputs, bf16
gradients), as for the unfused path, in every branch: with raw q/k, a chunk
whose decay span exceeds the single pivot runs the boundary-pivot path in fp32
on fp32 copies of q^, k^ and the other inputs.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
GRADS = ["dq", "dk", "dv", "dg", "de", "dw", "dgamma"]
TOL_FWD, TOL_BWD = 2e-3, 5e-3


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


def case(wid, over, gate, raw):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.fused_inputs(wid, with_dO=True, **over)
    args = dict(x)
    if raw:
        args["q"], args["k"] = x["xq"], x["xk"]
    z = x["z_out"] if gate else None
    return x, args, z


def run_oracle(orc, args, z, raw, dSf):
    og, S, o = orc.fwd_fused(*[args[n] for n in NAMES], S0=args["S0"], z_out=z, qk_raw=raw)
    gr = orc.bwd_fused(*[args[n] for n in NAMES], S0=args["S0"], dO=args["dO"], dS_final=dSf,
                       z_out=z, qk_raw=raw)
    return og, S, o, gr


CASES = [  # (workload id, overrides, output gate, raw q/k)
    (2, dict(B=1, H=2, T=512, s0_std=1.0), True, False),
    (2, dict(B=1, H=2, T=512, s0_std=1.0), False, True),
    (2, dict(B=2, H=2, T=384, s0_std=1.0), True, True),
    (3, dict(B=1, H=2, T=512), True, False),  # large decay spans: the fallback path
    (3, dict(B=1, H=2, T=512), True, True),   # the same, with raw q/k
]


@pytest.mark.parametrize("wid,over,gate,raw", CASES)
@pytest.mark.parametrize("saved", [True, False])
def test_fused_parity(muir, oracle_mod, wid, over, gate, raw, saved):
    x, args, z = case(wid, over, gate, raw)
    gen = torch.Generator().manual_seed(11)
    dSf = torch.randn(x["q"].shape[0], x["q"].shape[2], 128, 128, generator=gen)
    d = {n: (t.cuda() if t is not None else None) for n, t in args.items()}
    zd = z.cuda() if z is not None else None
    o, S, sv = muir.chunk_fwd_fused(*[d[n] for n in NAMES], d["S0"], z_out=zd, qk_raw=raw,
                                    out_dtype=torch.float32, save=saved)
    o_pre = sv["o_pre"] if saved else None
    if not saved and gate:  # the gated backward needs the forward's pre-gate output
        _, _, sv2 = muir.chunk_fwd_fused(*[d[n] for n in NAMES], d["S0"], z_out=zd, qk_raw=raw,
                                         out_dtype=torch.float32, save=True)
        o_pre = sv2["o_pre"]
    gr = muir.chunk_bwd_fused(*[d[n] for n in NAMES], d["S0"], d["dO"], dS_final=dSf.cuda(),
                              z_out=zd, qk_raw=raw, o_pre=o_pre, saved=sv if saved else None)
    torch.cuda.synchronize()
    og_r, S_r, o_r, gr_r = run_oracle(oracle_mod, args, z, raw, dSf)
    errs = {"o": nmax(o, og_r), "S": nmax(S, S_r)}
    if gate and o_pre is not None:
        errs["o_pre"] = nmax(o_pre, o_r)
    names = GRADS + ["dS0"] + (["dz_out"] if gate else [])
    errs.update({n: nmax(gr[n], gr_r[n]) for n in names})
    print(f"fused wid={wid} {over} gate={gate} raw={raw} saved={saved}: " +
          " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    for n in ("o", "S", "o_pre"):
        if n in errs:
            assert errs[n] < TOL_FWD, (n, errs)
    for n in names:
        assert errs[n] < TOL_BWD, (n, errs)


def test_fused_off_equals_plain_path(muir):
    """With both stages off the fused entry points run the plain path: the
    same bits as muir_chunk_fwd / muir_chunk_bwd."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2, B=1, H=2, T=256, with_dO=True)
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    o1, S1 = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128)
    o2, S2, _ = muir.chunk_fwd_fused(*[d[n] for n in NAMES], d["S0"], save=False)
    g1 = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], chunk=128)
    g2 = muir.chunk_bwd_fused(*[d[n] for n in NAMES], d["S0"], d["dO"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for n in GRADS + ["dS0"]:
        assert torch.equal(g1[n], g2[n]), n


def test_fused_refuses_unsupported_shapes(muir):
    """A fused stage on a shape the on-chip path does not take is refused on
    the host (MUIR_ERR_UNSUPPORTED) with real buffers of the shape's size."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.fused_inputs(0, dtype="bf16", B=1, H=2, T=200, dk=128, dv=128, with_dO=True)
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    with pytest.raises(muir.MuirError) as ei:
        muir.chunk_fwd_fused(*[d[n] for n in NAMES], d["S0"], z_out=d["z_out"], save=False)
    assert "UNSUPPORTED" in str(ei.value)
