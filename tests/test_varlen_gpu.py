"""Packed variable-length sequences (muir_chunk_fwd_varlen / muir_chunk_bwd_varlen)
against the fp64 oracle run on each sequence alone.

Sequences of mixed length share one token-major buffer [1, T, H, d]; each has its
own initial state and final state.  The lengths cover an empty sequence, a single
token, sequences shorter than one chunk, whole chunks and ragged tails.  Tolerances
as for the fixed-length path: 2e-3 (bf16) and 1e-5 (fp32) on o and S_final,
5e-3 / 1e-5 on gradients.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
TOL_FWD = {"bf16": 2e-3, "fp32": 1e-5}
TOL_BWD = {"bf16": 5e-3, "fp32": 1e-5}


@pytest.fixture(scope="module")
def muir():
    import gated_delta_rule_115_b200 as m
    m.lib()
    return m


def nmax(a, r):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


def packed(lengths, dtype, d, seed):
    from gated_delta_rule_115_b200 import inputs as I
    T = sum(lengths)
    x = I.chunk_inputs(0, dtype=dtype, T=T, H=2, dk=d, dv=d, s0_std=0.0, with_dO=True, seed=seed)
    n = len(lengths)
    g = torch.Generator().manual_seed(seed + 1)
    S0 = torch.randn(n, 2, d, d, generator=g)
    dSf = torch.randn(n, 2, d, d, generator=g)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return x, S0, dSf, cu


def seq(x, cu, i):
    return {k: (v[:, cu[i]:cu[i + 1]] if v is not None and v.dim() == 4 and k != "S0" else v)
            for k, v in x.items()}


CASES = [
    ([37, 0, 128, 1, 300, 64], "bf16", 128, 64),
    ([5, 250, 70], "fp32", 64, 64),
    ([200, 0, 129], "bf16", 64, 128),
    ([1, 2, 3], "fp32", 128, 16),
]


@pytest.mark.parametrize("lengths,dt,d,C", CASES)
def test_varlen_forward(muir, oracle_mod, lengths, dt, d, C):
    x, S0, _, cu = packed(lengths, dt, d, 40 + d + C)
    dev = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o, Sf = muir.chunk_fwd_varlen(*[dev[n] for n in NAMES], cu.tolist(), S0=S0.cuda(), chunk=C,
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    for i in range(len(lengths)):
        xi = seq(x, cu, i)
        if lengths[i] == 0:
            assert torch.equal(Sf[i].cpu(), S0[i])
            continue
        ro, rS = oracle_mod.fwd(*[xi[n] for n in NAMES], S0=S0[i:i + 1])
        eo, eS = nmax(o[:, cu[i]:cu[i + 1]], ro), nmax(Sf[i:i + 1], rS)
        print(f"varlen fwd seq {i} L={lengths[i]} {dt}: o {eo:.2e} S {eS:.2e}")
        assert eo < TOL_FWD[dt] and eS < TOL_FWD[dt]


@pytest.mark.parametrize("lengths,dt,d,C", CASES)
def test_varlen_backward(muir, oracle_mod, lengths, dt, d, C):
    x, S0, dSf, cu = packed(lengths, dt, d, 50 + d + C)
    dev = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    gr = muir.chunk_bwd_varlen(*[dev[n] for n in NAMES], cu.tolist(), S0.cuda(), dev["dO"],
                               dSf.cuda(), chunk=C)
    torch.cuda.synchronize()
    for i in range(len(lengths)):
        xi = seq(x, cu, i)
        if lengths[i] == 0:
            assert torch.equal(gr["dS0"][i].cpu(), dSf[i])
            continue
        rg = oracle_mod.bwd(*[xi[n] for n in NAMES], S0=S0[i:i + 1], dO=xi["dO"],
                            dS_final=dSf[i:i + 1])
        errs = {n: nmax(gr["d" + n][:, cu[i]:cu[i + 1]], rg["d" + n]) for n in NAMES}
        errs["S0"] = nmax(gr["dS0"][i:i + 1], rg["dS0"])
        print(f"varlen bwd seq {i} L={lengths[i]} {dt}: " +
              " ".join(f"d{k} {v:.2e}" for k, v in errs.items()))
        for n, e in errs.items():
            assert e < TOL_BWD[dt], (i, n, e)


def test_varlen_equals_separate_calls(muir):
    """The packed call gives bit for bit what one fixed-length call per sequence gives."""
    x, S0, _, cu = packed([70, 128, 3], "bf16", 128, 7)
    dev = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o, Sf = muir.chunk_fwd_varlen(*[dev[n] for n in NAMES], cu.tolist(), S0=S0.cuda(), chunk=64)
    for i in range(3):
        xi = seq(dev, cu, i)
        oi, Si = muir.chunk_fwd(*[xi[n].contiguous() for n in NAMES], S0[i:i + 1].cuda().contiguous(),
                                chunk=64)
        assert torch.equal(oi, o[:, cu[i]:cu[i + 1]])
        assert torch.equal(Si[0], Sf[i])
