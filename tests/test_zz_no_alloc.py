"""muir_chunk_fwd_noalloc: the chunkwise forward for callers that cannot
allocate device memory (its workspace lives in a fixed 16 MiB array inside the
library).  It must agree with muir_chunk_fwd, which uses a caller workspace,
on two calls in a row (the second call reuses whatever the first left in the
shared array), match the fp64 oracle, and reject shapes whose workspace does
not fit.  Every call gets real device buffers of its shape's size.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]
TOL = {"bf16": 2e-3, "fp32": 1e-5}


def nmax(a, r):
    a = a.double().cpu().numpy()
    r = r.double().cpu().numpy() if hasattr(r, "cpu") else np.asarray(r)
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


def call_noalloc(m, L, shp, d, o, S):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    S0 = ctypes.c_void_p(d["S0"].data_ptr()) if d.get("S0") is not None else None
    return L.muir_chunk_fwd_noalloc(ctypes.byref(shp), *[ctypes.c_void_p(d[n].data_ptr()) for n in NAMES],
                                    S0, ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(S.data_ptr()),
                                    stream)


@pytest.mark.parametrize("dtype,T", [("bf16", 256), ("fp32", 256), ("bf16", 250)])
def test_noalloc_forward_matches_workspace_forward(dtype, T, oracle_mod):
    import gated_delta_rule_115_b200 as m
    from gated_delta_rule_115_b200 import inputs as I
    L = m.lib()
    x = I.chunk_inputs(0, dtype=dtype, T=T, s0_std=1.0)
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o_ref, S_ref = m.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=64, out_dtype=torch.float32)
    ro, rS = oracle_mod.fwd(*[x[n] for n in NAMES], S0=x["S0"])
    B, T, H, dk = d["q"].shape
    shp = m.MuirShape(B, T, H, dk, dk, 64, m.MUIR_BF16 if dtype == "bf16" else m.MUIR_FP32,
                      m.MUIR_FP32)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = call_noalloc(m, L, shp, d, o, S)
        assert rc == 0, L.muir_status_string(rc)
        torch.cuda.synchronize()
        assert nmax(o, o_ref) < TOL[dtype], (call, nmax(o, o_ref))
        assert nmax(S, S_ref) < TOL[dtype], (call, nmax(S, S_ref))
        if call == 1:  # stands on its own against the oracle too
            assert nmax(o, ro) < TOL[dtype] and nmax(S, rS) < TOL[dtype]


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import gated_delta_rule_115_b200 as m
    from gated_delta_rule_115_b200 import inputs as I
    L = m.lib()
    # a shape whose workspace exceeds 16 MiB, with real buffers of its size
    x = I.chunk_inputs(2, B=1, H=2, T=1024, s0_std=1.0)
    big = m.MuirShape(1, 1024, 2, 128, 128, 64, m.MUIR_BF16, m.MUIR_FP32)
    assert L.muir_chunk_fwd_workspace(ctypes.byref(big)) > (16 << 20)
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o = torch.zeros(1, 1024, 2, 128, device="cuda")
    S = torch.zeros(1, 2, 128, 128, device="cuda")
    assert call_noalloc(m, L, big, d, o, S) == 3  # MUIR_ERR_WORKSPACE
    # an unsupported head dim is refused before anything is enqueued
    y = I.chunk_inputs(0, dtype="bf16", B=1, H=2, T=256, dk=96, dv=96)
    dy = {k: (v.cuda() if v is not None else None) for k, v in y.items()}
    bad = m.MuirShape(1, 256, 2, 96, 96, 64, m.MUIR_BF16, m.MUIR_FP32)
    o2 = torch.zeros(1, 256, 2, 96, device="cuda")
    S2 = torch.zeros(1, 2, 96, 96, device="cuda")
    assert call_noalloc(m, L, bad, dy, o2, S2) == 2  # MUIR_ERR_UNSUPPORTED
    torch.cuda.synchronize()
