"""Parity of the CUDA chunkwise forward/backward (muir_chunk_fwd / muir_chunk_bwd)
against the fp64 oracle, on seeded inputs from gated_delta_rule_115_b200.inputs.

Error metric (one number per tensor): max |gpu - oracle| / max |oracle|.
Tolerances: o and S_final 2e-3 for bf16 inputs and 1e-5 for float32 inputs;
gradients 5e-3 (bf16) and 1e-5 (float32).  Both sides read the same values:
the oracle upcasts the exact bf16/fp32 inputs to float64.  Heads are
independent, so at full sizes a sampled subset of (b, h) is checked exactly.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
TOL_FWD = {"bf16": 2e-3, "fp32": 1e-5}
TOL_BWD = {"bf16": 5e-3, "fp32": 1e-5}


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
    """Every test ends with no expired bounded wait in any chunk kernel."""
    muir.device_wait_status()
    yield
    muir.device_wait_status()


def to_dev(x):
    return {k: (v.cuda() if v is not None else None) for k, v in x.items()}


def sub(x, bs, hs):
    """Select batches bs and heads hs of every tensor (oracle side, CPU)."""
    out = {}
    for k, v in x.items():
        if v is None:
            out[k] = None
        elif v.dim() == 4 and k != "S0":
            out[k] = v[bs][:, :, hs]
        else:  # S0 [B,H,dk,dv]
            out[k] = v[bs][:, hs]
    return out


CASES = [
    # (wid, overrides, chunk)
    (0, dict(), 64),                                             # tiny fp32 forward workload
    (0, dict(dtype="bf16", T=128, dk=128, dv=128, s0_std=1.0), 16),
    (0, dict(dtype="bf16", T=256, dk=128, dv=128, s0_std=1.0), 32),
    (1, dict(B=2, H=2, T=512, gates="proj"), 64),
    (2, dict(B=1, H=2, T=512), 128),
    (3, dict(B=1, H=2, T=1024), 256),
    (0, dict(dtype="fp32", T=256, dk=128, dv=128, s0_std=2.0), 128),
    (0, dict(dtype="bf16", T=192, dk=64, dv=64, s0_std=1.0), 64),
]


@pytest.mark.parametrize("wid,over,C", CASES)
def test_chunk_fwd_parity(muir, oracle_mod, wid, over, C):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    dt = over.get("dtype", I.WORKLOADS[wid].dtype)
    d = to_dev(x)
    o, S, Sc = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=C, out_dtype=torch.float32,
                              return_chunk_states=True)
    ro, rS, rSc = oracle_mod.chunk_fwd(*[x[n] for n in NAMES], S0=x["S0"], chunk=C)
    torch.cuda.synchronize()
    eo, eS, eC = nmax(o, ro), nmax(S, rS), nmax(Sc, rSc)
    print(f"fwd wid={wid} C={C} {dt}: o {eo:.2e} S {eS:.2e} chunk states {eC:.2e}")
    assert eo < TOL_FWD[dt] and eS < TOL_FWD[dt] and eC < TOL_FWD[dt]


def test_chunk_fwd_bf16_output(muir):
    from gated_delta_rule_115_b200 import inputs as I
    x = to_dev(I.chunk_inputs(2, B=1, H=2, T=256))
    o32, _ = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128, out_dtype=torch.float32)
    o16, _ = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128, out_dtype=torch.bfloat16)
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_chunk_fwd_decay_below_clamp(muir, oracle_mod):
    """Log decays far below the kernels' clamp (-20) still match: a row decayed
    by exp(-20) or more is erased either way."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(0, dtype="fp32", T=128, s0_std=3.0)
    x["g"] = x["g"] * 30.0 - 5.0  # values down to about -150
    d = to_dev(x)
    o, S = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=64, out_dtype=torch.float32)
    ro, rS = oracle_mod.fwd(*[x[n] for n in NAMES], S0=x["S0"])
    torch.cuda.synchronize()
    assert np.isfinite(o.cpu().numpy()).all()
    assert nmax(o, ro) < 1e-5 and nmax(S, rS) < 1e-5


def test_chunk_size_invariance_on_gpu(muir):
    """The GPU results for C = 16 ... 256 agree with each other (same inputs)."""
    from gated_delta_rule_115_b200 import inputs as I
    x = to_dev(I.chunk_inputs(0, dtype="fp32", T=512, dk=64, dv=64, s0_std=1.0))
    outs = [muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=C, out_dtype=torch.float32)
            for C in (16, 32, 64, 128, 256)]
    ref = outs[-1][0].double().cpu().numpy()
    for o, S in outs[:-1]:
        assert nmax(o, ref) < 1e-5


BWD_CASES = [
    (0, dict(s0_std=1.0), 64),                                    # fp32, d=64
    (2, dict(B=1, H=2, T=512), 128),                              # long-context slice, bf16
    (1, dict(B=1, H=2, T=256, with_dO=True, s0_std=1.0), 64),
    (3, dict(B=1, H=1, T=512, with_dO=True), 256),
    (0, dict(dtype="bf16", T=64, dk=128, dv=128, s0_std=1.0), 16),
    (0, dict(dtype="fp32", T=256, dk=128, dv=128, s0_std=1.0), 32),
]


@pytest.mark.parametrize("wid,over,C", BWD_CASES)
def test_chunk_bwd_parity(muir, oracle_mod, wid, over, C):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    dt = over.get("dtype", I.WORKLOADS[wid].dtype)
    B, T, H, dk = x["q"].shape
    gen = torch.Generator().manual_seed(99)
    dSf = torch.randn(B, H, dk, dk, generator=gen)
    d = to_dev(x)
    gr = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], dSf.cuda(), chunk=C)
    rg = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"], dS_final=dSf)
    torch.cuda.synchronize()
    errs = {n: nmax(gr["d" + n], rg["d" + n]) for n in NAMES}
    errs["S0"] = nmax(gr["dS0"], rg["dS0"])
    print(f"bwd wid={wid} C={C} {dt}: " + " ".join(f"d{k} {v:.2e}" for k, v in errs.items()))
    for n, e in errs.items():
        assert e < TOL_BWD[dt], (n, e)


def test_chunk_bwd_reuses_states(muir):
    """Passing the forward's chunk states to the backward gives the same
    gradients as recomputing them."""
    from gated_delta_rule_115_b200 import inputs as I
    x = to_dev(I.chunk_inputs(2, B=1, H=2, T=512, s0_std=1.0))
    o, S, Sc = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128, return_chunk_states=True)
    a = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128)
    b = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128, S_chunks=Sc)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    # with the transitions as well, the backward skips recomputing them
    o2, S2, Sc2, Mc2 = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128, return_saved=True)
    assert torch.equal(Sc2, Sc) and torch.equal(o2, o)
    c = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128, S_chunks=Sc2,
                       M_chunks=Mc2)
    for k in a:
        assert torch.equal(a[k], c[k]), k
    # with the saved intermediates too, the backward skips the masked products,
    # the block inverses and Y, and the result does not change
    o3, S3, Sc3, Mc3, aux = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128,
                                           return_saved=True, save_aux=True)
    assert torch.equal(o3, o) and torch.equal(Sc3, Sc)
    e = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128, S_chunks=Sc3,
                       M_chunks=Mc3, aux=aux)
    for k in a:
        assert torch.equal(a[k], e[k]), k


# ------------------------------------------------- span-dependent product paths

# Chunks whose per-channel log decay over the chunk stays within 140 take
# single-pivot products; larger spans take the 8-token pivoted panels.  These
# cases scale g so that every chunk, or every other chunk, needs the panels.
SPAN_CASES = [
    ("all-panels", 3.0, None),
    ("mixed", 3.0, 2),
]


def _span_inputs(scale, every):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2, B=1, H=2, T=512, s0_std=1.0)
    g = x["g"].float()
    if every is None:
        g = g * scale
    else:  # scale the tokens of every other 128-token chunk
        T = g.shape[1]
        idx = torch.arange(T) // 128
        sel = (idx % every == 0).view(1, T, 1, 1)
        g = torch.where(sel, g * scale, g)
    x["g"] = g.to(x["g"].dtype)
    return x


@pytest.mark.parametrize("name,scale,every", SPAN_CASES)
def test_chunk_fwd_span_paths(muir, oracle_mod, name, scale, every):
    x = _span_inputs(scale, every)
    d = to_dev(x)
    o, S, Sc = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128, out_dtype=torch.float32,
                              return_chunk_states=True)
    ro, rS, rSc = oracle_mod.chunk_fwd(*[x[n] for n in NAMES], S0=x["S0"], chunk=128)
    torch.cuda.synchronize()
    eo, eS, eC = nmax(o, ro), nmax(S, rS), nmax(Sc, rSc)
    print(f"fwd span {name}: o {eo:.2e} S {eS:.2e} chunk states {eC:.2e}")
    assert eo < TOL_FWD["bf16"] and eS < TOL_FWD["bf16"] and eC < TOL_FWD["bf16"]


@pytest.mark.parametrize("name,scale,every", SPAN_CASES)
def test_chunk_bwd_span_paths(muir, oracle_mod, name, scale, every):
    x = _span_inputs(scale, every)
    B, T, H, dk = x["q"].shape
    dSf = torch.randn(B, H, dk, dk, generator=torch.Generator().manual_seed(7))
    d = to_dev(x)
    gr = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], dSf.cuda(), chunk=128)
    rg = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"], dS_final=dSf)
    torch.cuda.synchronize()
    errs = {n: nmax(gr["d" + n], rg["d" + n]) for n in NAMES}
    errs["S0"] = nmax(gr["dS0"], rg["dS0"])
    print(f"bwd span {name}: " + " ".join(f"d{k} {v:.2e}" for k, v in errs.items()))
    for n, e in errs.items():
        assert e < TOL_BWD["bf16"], (n, e)
    # the saved-intermediates path gives the same gradients on both product paths
    o, S, Sc, Mc, aux = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128,
                                       return_saved=True, save_aux=True)
    gs = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], dSf.cuda(), chunk=128,
                        S_chunks=Sc, M_chunks=Mc, aux=aux)
    for k in gr:
        assert torch.equal(gr[k], gs[k]), k


# ------------------------------------------------------------ ragged tails

# T not a multiple of C: the last chunk holds the remaining tokens (down to a
# single one, and T < C where the whole sequence is one partial chunk).
RAGGED_FWD = [
    # (wid, overrides, chunk)
    (0, dict(T=250), 64),                                         # fp32 d=64, tail 58
    (0, dict(dtype="bf16", T=200, dk=128, dv=128, s0_std=1.0), 128),
    (2, dict(B=2, H=2, T=300), 128),                              # batch stride, tail 44
    (0, dict(dtype="fp32", T=37, dk=128, dv=128, s0_std=1.0), 64),  # T < C
    (0, dict(dtype="bf16", T=1, s0_std=1.0), 16),                 # one token
    (3, dict(B=1, H=2, T=700), 256),                              # tail 188
    (0, dict(dtype="fp32", T=130, dk=128, dv=128, s0_std=2.0), 32),  # tail 2
]


@pytest.mark.parametrize("wid,over,C", RAGGED_FWD)
def test_chunk_fwd_ragged_tail(muir, oracle_mod, wid, over, C):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    dt = over.get("dtype", I.WORKLOADS[wid].dtype)
    d = to_dev(x)
    o, S, Sc = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=C, out_dtype=torch.float32,
                              return_chunk_states=True)
    ro, rS, rSc = oracle_mod.chunk_fwd(*[x[n] for n in NAMES], S0=x["S0"], chunk=C)
    torch.cuda.synchronize()
    assert Sc.shape[2] == -(-x["q"].shape[1] // C)
    eo, eS, eC = nmax(o, ro), nmax(S, rS), nmax(Sc, rSc)
    print(f"ragged fwd wid={wid} C={C} {dt}: o {eo:.2e} S {eS:.2e} chunk states {eC:.2e}")
    assert eo < TOL_FWD[dt] and eS < TOL_FWD[dt] and eC < TOL_FWD[dt]


RAGGED_BWD = [
    (0, dict(T=250, s0_std=1.0), 64),
    (2, dict(B=2, H=2, T=300), 128),
    (0, dict(dtype="bf16", T=37, dk=128, dv=128, s0_std=1.0), 64),
    (3, dict(B=1, H=1, T=600, with_dO=True), 256),
    (0, dict(dtype="fp32", T=130, dk=128, dv=128, s0_std=1.0), 32),
]


@pytest.mark.parametrize("wid,over,C", RAGGED_BWD)
def test_chunk_bwd_ragged_tail(muir, oracle_mod, wid, over, C):
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid, **over)
    dt = over.get("dtype", I.WORKLOADS[wid].dtype)
    B, T, H, dk = x["q"].shape
    dSf = torch.randn(B, H, dk, dk, generator=torch.Generator().manual_seed(98))
    d = to_dev(x)
    gr = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], dSf.cuda(), chunk=C)
    rg = oracle_mod.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"], dS_final=dSf)
    torch.cuda.synchronize()
    errs = {n: nmax(gr["d" + n], rg["d" + n]) for n in NAMES}
    errs["S0"] = nmax(gr["dS0"], rg["dS0"])
    print(f"ragged bwd wid={wid} C={C} {dt}: " + " ".join(f"d{k} {v:.2e}" for k, v in errs.items()))
    for n, e in errs.items():
        assert e < TOL_BWD[dt], (n, e)


def test_ragged_tail_reuses_saved(muir):
    """With a ragged tail, the backward from the forward's saved states,
    transitions and intermediates equals the recomputing backward bit for bit,
    and the forward equals the one over the sequences zero-padded by hand."""
    from gated_delta_rule_115_b200 import inputs as I
    x = to_dev(I.chunk_inputs(2, B=2, H=2, T=333, s0_std=1.0))
    a = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128)
    o, S, Sc, Mc, aux = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128,
                                       return_saved=True, save_aux=True)
    b = muir.chunk_bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], chunk=128, S_chunks=Sc,
                       M_chunks=Mc, aux=aux)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    # the same sequences padded by hand to 384 tokens with zero tokens give the
    # same o on the real rows and the same final state.  The padded call
    # (T a multiple of 128) runs the on-chip tensor-core path, the ragged one
    # the boundary-pivot path, so they agree within the forward tolerance
    # rather than bit for bit (o is bf16: one rounding step on each side).
    pad = {n: (torch.cat([x[n], torch.zeros_like(x[n][:, :51])], 1) if x[n].dim() == 4 and n != "S0"
               else x[n]) for n in NAMES + ["S0"]}
    op, Sp = muir.chunk_fwd(*[pad[n] for n in NAMES], pad["S0"], chunk=128, out_dtype=torch.float32)
    o32, S32 = muir.chunk_fwd(*[x[n] for n in NAMES], x["S0"], chunk=128, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref_o = o32.double().cpu().numpy()
    assert nmax(op[:, :333], ref_o) < 2 * TOL_FWD["bf16"]
    assert nmax(Sp, S32.double().cpu().numpy()) < 2 * TOL_FWD["bf16"]
    assert torch.equal(S32, S)


# ------------------------------------------------------------ full-size workloads

FULL = [(1, 64), (2, 128), (3, 256)]


@pytest.mark.parametrize("wid,C", FULL)
def test_full_size_forward_sampled_heads(muir, oracle_mod, wid, C):
    """Forward at the workload's full size (the launch configuration the bench
    times); o and S_final of sampled (b, h) against the oracle."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(wid)
    d = to_dev(x)
    o, S = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=C, out_dtype=torch.float32)
    torch.cuda.synchronize()
    B, T, H, _ = x["q"].shape
    rng = np.random.default_rng(wid)
    bs = sorted(rng.choice(B, min(B, 2), replace=False).tolist())
    hs = sorted(rng.choice(H, 2, replace=False).tolist())
    xs = sub(x, bs, hs)
    ro, rS = oracle_mod.fwd(*[xs[n] for n in NAMES], S0=xs["S0"])
    eo = nmax(o.cpu()[bs][:, :, hs], ro)
    eS = nmax(S.cpu()[bs][:, hs], rS)
    print(f"full fwd wid={wid}: o {eo:.2e} S {eS:.2e}")
    assert eo < 2e-3 and eS < 2e-3


def test_full_size_fwd_bwd_long_context(muir, oracle_mod):
    """The long-context workload (B=1, H=16, T=32768, d=128, C=128) through the
    forward (saving chunk states) and backward exactly as the bench runs it;
    gradients of one sampled head against the oracle's BPTT over the full length."""
    from gated_delta_rule_115_b200 import inputs as I
    x = I.chunk_inputs(2)
    d = to_dev(x)
    o, S, Sc, Mc, aux = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=128,
                                       return_saved=True, save_aux=True)
    gr = muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], chunk=128, S_chunks=Sc,
                        M_chunks=Mc, aux=aux)
    torch.cuda.synchronize()
    hs = [11]
    xs = sub(x, [0], hs)
    rg = oracle_mod.bwd(*[xs[n] for n in NAMES], S0=xs["S0"], dO=xs["dO"], ckpt=128)
    for n in NAMES:
        e = nmax(gr["d" + n].cpu()[:, :, hs], rg["d" + n])
        print(f"full bwd d{n}: {e:.2e}")
        assert e < 5e-3, (n, e)
