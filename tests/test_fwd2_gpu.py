"""Parity of the on-chip tensor-core forward (bf16 inputs, d = 128, chunk 128,
T a multiple of 128) against the fp64 oracle, and of its device-side switch to
the boundary-pivot path when a chunk's decay span exceeds the single pivot.

Metric: max |gpu - oracle| / max |oracle| per tensor; bound 2e-3 (bf16 inputs).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
TOL = 2e-3


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


def elem_rel(a, r):
    """Elementwise relative error with a floor of 1e-3 max|r| (the second
    metric of the parity reading: logged, and below 1, i.e. no element is off
    by as much as its own magnitude where that is above the floor)."""
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


CASES = [
    # (workload, overrides)
    (2, dict(B=1, H=2, T=512)),                         # projected gates, zero state
    (2, dict(B=2, H=3, T=384, s0_std=1.0)),             # several heads and batches, S0
    (0, dict(dtype="bf16", B=1, H=2, T=256, dk=128, dv=128, s0_std=2.0)),  # iid gates
    (2, dict(B=1, H=1, T=128)),                         # a single chunk
]


@pytest.mark.parametrize("wid,over", CASES)
def test_fwd2_parity(muir, oracle_mod, wid, over):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    d = to_dev(x)
    o, S, Sc = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128,
                              out_dtype=torch.float32, return_chunk_states=True)
    ro, rS, rSc = oracle_mod.chunk_fwd(*[x[n] for n in NAMES], S0=x["S0"], chunk=128)
    torch.cuda.synchronize()
    eo, eS, eC = nmax(o, ro), nmax(S, rS), nmax(Sc, rSc)
    lo, lS = elem_rel(o, ro), elem_rel(S, rS)
    print(f"fwd2 wid={wid} {over}: o {eo:.2e} S {eS:.2e} chunk states {eC:.2e}; "
          f"elementwise (floor 1e-3 max): o {lo:.2e} S {lS:.2e}")
    assert eo < TOL and eS < TOL and eC < TOL
    assert lo < 1.0 and lS < 1.0


def test_fwd2_many_chunks_per_cta(muir, oracle_mod):
    """More chunks than SMs: every persistent CTA loops over several chunks.
    Sampled heads are checked against the oracle."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2, B=1, H=16, T=2048)
    d = to_dev(x)
    o, S = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for h in (0, 7, 15):
        xs = {n: x[n][:, :, h:h + 1] for n in NAMES}
        ro, rS = oracle_mod.fwd(*[xs[n] for n in NAMES])
        eo, eS = nmax(o[:, :, h:h + 1], ro), nmax(S[:, h:h + 1], rS)
        print(f"head {h}: o {eo:.2e} S {eS:.2e}")
        assert eo < TOL and eS < TOL


@pytest.mark.parametrize("mixed", [False, True])
def test_fwd2_large_span_switch(muir, oracle_mod, mixed):
    """Chunks whose decay summed over 128 tokens is below -140 in some channel
    are outside the single pivot; the device flag then runs the boundary-pivot
    path, which must give the oracle's result.  mixed: only one chunk of one
    head decays that fast."""
    from gated_delta_rule_115_b200 import inputs as I
    if mixed:
        x = I.chunk_inputs(2, B=1, H=2, T=512, s0_std=1.0)
        g = x["g"].float()
        g[0, 256:384, 1, 5] = -3.0  # span 384 in one channel of one chunk
        x["g"] = g.to(torch.bfloat16)
    else:
        x = I.chunk_inputs(3, B=1, H=2, T=512)
    d = to_dev(x)
    o, S = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128, out_dtype=torch.float32)
    ro, rS = oracle_mod.fwd(*[x[n] for n in NAMES], S0=x["S0"])
    torch.cuda.synchronize()
    eo, eS = nmax(o, ro), nmax(S, rS)
    print(f"large span (mixed={mixed}): o {eo:.2e} S {eS:.2e}")
    assert eo < TOL and eS < TOL
