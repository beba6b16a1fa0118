"""Parity of the on-chip tensor-core backward (bf16 inputs, d = 128, chunk 128,
T a multiple of 128) against the fp64 oracle's back-propagation through time,
with the forward's saved intermediates and with a recomputed forward, and of
the device-side switch to the boundary-pivot path for large decay spans.

Metric: max |gpu - oracle| / max |oracle| per gradient tensor; bound 5e-3
(bf16 inputs, gradients stored in bf16).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
GRADS = ["dq", "dk", "dv", "dg", "de", "dw", "dgamma"]
TOL = 5e-3


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


def elem_rel(a, r):
    """Elementwise relative error with a floor of 1e-3 max|r|: logged, with only a
    sanity bound of 2 (dg is a suffix sum over the chunk, and entries just above
    the floor after cancellation carry the error of the large terms)."""
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    r = np.asarray(r)
    floor = 1e-3 * max(np.abs(r).max(), 1e-300)
    return float((np.abs(a - r) / np.maximum(np.abs(r), floor)).max())


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


def to_dev(x):
    return {k: (v.cuda() if v is not None else None) for k, v in x.items()}


def run_bwd(muir, x, saved, dSf=None):
    d = to_dev(x)
    args = [d[n] for n in NAMES]
    dSf_d = dSf.cuda() if dSf is not None else None
    if saved:
        _, _, Sc, Mc, aux = muir.chunk_fwd(*args, d["S0"], chunk=128, return_saved=True,
                                           save_aux=True)
        return muir.chunk_bwd(*args, d["S0"], d["dO"], dS_final=dSf_d, chunk=128, S_chunks=Sc,
                              M_chunks=Mc, aux=aux)
    return muir.chunk_bwd(*args, d["S0"], d["dO"], dS_final=dSf_d, chunk=128)


CASES = [
    (2, dict(B=1, H=2, T=512), False),
    (2, dict(B=1, H=2, T=512, s0_std=1.0), True),
    (2, dict(B=2, H=3, T=384, s0_std=1.0), True),
    (0, dict(dtype="bf16", B=1, H=2, T=256, dk=128, dv=128, s0_std=2.0, with_dO=True), True),
    (2, dict(B=1, H=1, T=128), True),
]


@pytest.mark.parametrize("wid,over,saved", CASES)
def test_bwd2_parity(muir, oracle_mod, wid, over, saved):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    gen = torch.Generator().manual_seed(7)
    dSf = torch.randn(x["q"].shape[0], x["q"].shape[2], 128, 128, generator=gen)
    gr = run_bwd(muir, x, saved, dSf)
    ref = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"], dS_final=dSf)
    torch.cuda.synchronize()
    errs = {n: nmax(gr[n], ref[n]) for n in GRADS + ["dS0"]}
    elem = {n: elem_rel(gr[n], ref[n]) for n in GRADS + ["dS0"]}
    print(f"bwd2 wid={wid} {over} saved={saved}: " + " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    print("  elementwise (floor 1e-3 max): " + " ".join(f"{n} {v:.2e}" for n, v in elem.items()))
    assert all(v < TOL for v in errs.values()), errs
    assert all(v < 2.0 for v in elem.values()), elem


def test_bwd2_many_chunks_per_cta(muir, oracle_mod):
    """More chunks than SMs; sampled heads against the oracle."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2, B=1, H=16, T=2048)
    gr = run_bwd(muir, x, True)
    torch.cuda.synchronize()
    for h in (0, 9):
        xs = {n: x[n][:, :, h:h + 1] for n in NAMES + ["dO"]}
        ref = oracle_mod.bwd(*[xs[n] for n in NAMES], dO=xs["dO"])
        errs = {n: nmax(gr[n][:, :, h:h + 1], ref[n]) for n in GRADS}
        print(f"head {h}: " + " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
        assert all(v < TOL for v in errs.values()), errs


def test_bwd2_large_span_switch(muir, oracle_mod):
    """Decays beyond the single pivot run the boundary-pivot backward."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(3, B=1, H=2, T=512, with_dO=True)
    gr = run_bwd(muir, x, True)
    ref = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"])
    torch.cuda.synchronize()
    errs = {n: nmax(gr[n], ref[n]) for n in GRADS + ["dS0"]}
    print("large span: " + " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    assert all(v < TOL for v in errs.values()), errs
