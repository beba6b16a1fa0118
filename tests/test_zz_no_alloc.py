"""muir_chunk_fwd_noalloc: the chunkwise forward for callers that cannot
allocate device memory (its workspace lives in a fixed 16 MiB array inside the
library).  It must agree with muir_chunk_fwd, which uses a caller workspace,
on two calls in a row (the second call reuses whatever the first left in the
shared array), and reject shapes whose workspace does not fit.

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
    r = r.double().cpu().numpy()
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


@pytest.mark.parametrize("dtype,T", [("bf16", 256), ("fp32", 256), ("bf16", 250)])
def test_noalloc_forward_matches_workspace_forward(dtype, T):
    import gated_delta_rule_115_b200 as m
    from gated_delta_rule_115_b200 import inputs as I
    L = m.lib()
    x = I.chunk_inputs(0, dtype=dtype, T=T, s0_std=1.0)
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o_ref, S_ref = m.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=64, out_dtype=torch.float32)
    B, T, H, dk = d["q"].shape
    shp = m.MuirShape(B, T, H, dk, dk, 64, m.MUIR_BF16 if dtype == "bf16" else m.MUIR_FP32,
                      m.MUIR_FP32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = L.muir_chunk_fwd_noalloc(ctypes.byref(shp), *[ctypes.c_void_p(d[n].data_ptr()) for n in NAMES],
                                      ctypes.c_void_p(d["S0"].data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                      ctypes.c_void_p(S.data_ptr()), stream)
        assert rc == 0, L.muir_status_string(rc)
        torch.cuda.synchronize()
        assert nmax(o, o_ref) < TOL[dtype], (call, nmax(o, o_ref))
        assert nmax(S, S_ref) < TOL[dtype], (call, nmax(S, S_ref))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import gated_delta_rule_115_b200 as m
    L = m.lib()
    big = m.MuirShape(1, 32768, 16, 128, 128, 128, m.MUIR_BF16, m.MUIR_FP32)
    assert L.muir_chunk_fwd_workspace(ctypes.byref(big)) > (16 << 20)
    fake = ctypes.c_void_p(0x10000)
    rc = L.muir_chunk_fwd_noalloc(ctypes.byref(big), *([fake] * 7), None, fake, None, None)
    assert rc == 3  # MUIR_ERR_WORKSPACE
    # fake pointers only ever go with shapes the host checks reject: nothing is launched
    bad = m.MuirShape(1, 256, 2, 96, 96, 64, m.MUIR_BF16, m.MUIR_FP32)
    assert L.muir_chunk_fwd_noalloc(ctypes.byref(bad), *([fake] * 7), None, fake, None, None) == 2
