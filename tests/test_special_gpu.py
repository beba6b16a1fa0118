"""GPU parity of the special cases the recurrence reduces to ("Muir",
wolonglab.org page, "Methodology": decay, erase and write gates of the gated
delta rule), run through the on-chip path (bf16, dk = dv = 128, chunk
128), forward and backward, against the fp64 oracle, whose own pins fix these
cases to closed forms:

* e = 0, g = 0: plain linear attention (no decay, no erase); g = 0 is also the
  zero-span case of the single decay pivot;
* g = 0, e = w = 1: the delta rule (Widrow-Hoff with unit step and unit keys);

and of the bounded-wait self-test: a device wait that runs out is reported by
muir_device_wait_status as MUIR_ERR_DEVICE_TIMEOUT, without a fault.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
GRADS = ["dq", "dk", "dv", "dg", "de", "dw", "dgamma"]


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


@pytest.fixture(scope="module")
def muir():
    import gated_delta_rule_115_b200 as m
    m.lib()
    return m


def special(kind):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2, B=1, H=2, T=512, s0_std=1.0, with_dO=True)
    x["g"] = torch.zeros_like(x["g"])
    if kind == "linear_attention":
        x["e"] = torch.zeros_like(x["e"])
    else:  # delta rule
        x["e"] = torch.ones_like(x["e"])
        x["w"] = torch.ones_like(x["w"])
    return x


@pytest.mark.parametrize("kind", ["linear_attention", "delta_rule"])
def test_special_case_parity(muir, oracle_mod, kind):
    x = special(kind)
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    args = [d[n] for n in NAMES]
    o, S, Sc, Mc, aux = muir.chunk_fwd(*args, d["S0"], chunk=128, out_dtype=torch.float32,
                                       return_saved=True, save_aux=True)
    gr = muir.chunk_bwd(*args, d["S0"], d["dO"], chunk=128, S_chunks=Sc, M_chunks=Mc, aux=aux)
    torch.cuda.synchronize()
    muir.device_wait_status()
    ro, rS = oracle_mod.fwd(*[x[n] for n in NAMES], S0=x["S0"])
    rg = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"])
    errs = {"o": nmax(o, ro), "S": nmax(S, rS)}
    errs.update({n: nmax(gr[n], rg[n]) for n in GRADS + ["dS0"]})
    print(f"{kind}: " + " ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    assert errs["o"] < 2e-3 and errs["S"] < 2e-3, errs
    assert all(errs[n] < 5e-3 for n in GRADS + ["dS0"]), errs


def test_expired_wait_is_reported(muir):
    L = muir.lib()
    muir.device_wait_status()  # clear
    stream = torch.cuda.current_stream().cuda_stream
    assert L.muir_selftest_expired_wait(2000, stream) == 0
    assert L.muir_device_wait_status() == 5  # MUIR_ERR_DEVICE_TIMEOUT
    assert L.muir_device_wait_status() == 0  # the record was cleared
    x = torch.ones(4, device="cuda")         # the context is still usable
    assert float((x * 2).sum()) == 8.0
