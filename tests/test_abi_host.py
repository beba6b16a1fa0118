"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function ``include/muir.h`` declares, and
reject bad arguments with the documented status codes before touching CUDA.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_115_b200 import build
    build.build()
    import gated_delta_rule_115_b200 as m
    return m.lib()


def header_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
            names |= set(re.findall(r"\b(muir_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert {"muir_chunk_fwd", "muir_chunk_bwd", "muir_recurrent_step"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    assert "muir_profile_collect" in names


def test_profile_hook_without_launches(L):
    L.muir_profile_reset()
    L.muir_profile_enable(1)
    L.muir_profile_enable(0)
    assert L.muir_profile_collect() == 0
    assert L.muir_profile_count() == 0
    assert L.muir_profile_name(0) is None


def test_status_strings(L):
    for code in range(6):
        s = L.muir_status_string(code).decode()
        assert s.startswith("MUIR_")
    assert L.muir_status_string(99).decode() == "MUIR_ERR_UNKNOWN"


def _shape(m, **kw):
    d = dict(B=1, T=256, H=2, dk=64, dv=64, chunk=64, in_dtype=0, out_dtype=1)
    d.update(kw)
    return m.MuirShape(**d)


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: checks fail first


def _fwd(L, shp, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, e=FAKE, w=FAKE, gamma=FAKE, S0=None, o=FAKE,
                S_final=None, S_chunks=None, M_chunks=None, aux=None, ws=None, ws_bytes=0)
    args.update(over)
    return L.muir_chunk_fwd(ctypes.byref(shp), args["q"], args["k"], args["v"], args["g"],
                            args["e"], args["w"], args["gamma"], args["S0"], args["o"],
                            args["S_final"], args["S_chunks"], args["M_chunks"], args["aux"],
                            args["ws"], ctypes.c_size_t(args["ws_bytes"]), None)


def test_chunk_fwd_rejects_bad_arguments(L):
    import gated_delta_rule_115_b200 as m
    assert _fwd(L, _shape(m, dk=96, dv=96)) == 2            # head dim
    assert _fwd(L, _shape(m, dk=64, dv=128)) == 2           # dk != dv
    assert _fwd(L, _shape(m, chunk=48)) == 2                # chunk size
    assert _fwd(L, _shape(m, T=0)) == 1                     # empty sequence
    assert _fwd(L, _shape(m, T=250)) == 3                   # ragged tail: valid, needs workspace
    assert _fwd(L, _shape(m, B=0)) == 1
    assert _fwd(L, _shape(m, in_dtype=7)) == 1
    assert _fwd(L, _shape(m), q=None) == 1                  # null input
    assert _fwd(L, _shape(m), o=ctypes.c_void_p(0x10004)) == 1  # misaligned output
    assert _fwd(L, _shape(m), M_chunks=ctypes.c_void_p(0x10002)) == 1  # misaligned saved array
    assert _fwd(L, _shape(m), aux=ctypes.c_void_p(0x10004)) == 1       # misaligned intermediates
    assert L.muir_chunk_fwd(None, *([FAKE] * 14), ctypes.c_size_t(0), None) == 1


def test_chunk_aux_size(L):
    import gated_delta_rule_115_b200 as m
    # per chunk: 4 C x C masked matrices, C x 16 block inverses, C x d for Y
    assert L.muir_chunk_aux_floats(ctypes.byref(_shape(m))) == 1 * 2 * 4 * (4 * 64 * 64 + 64 * 16 + 64 * 64)
    assert L.muir_chunk_aux_floats(ctypes.byref(_shape(m, chunk=48))) == 0
    # ceil(T / C) chunks with a ragged tail
    assert L.muir_chunk_aux_floats(ctypes.byref(_shape(m, T=250))) == \
        L.muir_chunk_aux_floats(ctypes.byref(_shape(m)))


def test_chunk_workspace_query(L):
    import gated_delta_rule_115_b200 as m
    assert L.muir_chunk_fwd_workspace(ctypes.byref(_shape(m, chunk=48))) == 0
    assert L.muir_chunk_bwd_workspace(ctypes.byref(_shape(m, T=0))) == 0
    # a ragged tail adds the side buffers of the padded last chunk
    # (8 inputs + 7 outputs of B*H*C*d elements, 4 bytes each)
    for q in (L.muir_chunk_fwd_workspace, L.muir_chunk_bwd_workspace):
        assert q(ctypes.byref(_shape(m, T=250))) == q(ctypes.byref(_shape(m))) + 15 * 2 * 64 * 64 * 4
    need = L.muir_chunk_fwd_workspace(ctypes.byref(_shape(m)))
    if need > 0:
        assert _fwd(L, _shape(m), ws=FAKE, ws_bytes=need - 1) == 3
        assert _fwd(L, _shape(m), ws=None, ws_bytes=need) == 3


def test_chunk_bwd_rejects_bad_arguments(L):
    import gated_delta_rule_115_b200 as m
    shp = _shape(m, dk=32, dv=32)
    # q k v g e w gamma | S0 S_chunks M_chunks aux | dO dS_final | dq .. dgamma | dS0 ws
    args = [FAKE] * 7 + [None, None, None, None, FAKE, None] + [FAKE] * 7 + [None, None]
    assert L.muir_chunk_bwd(ctypes.byref(shp), *args, ctypes.c_size_t(0), None) == 2
    shp = _shape(m)
    args2 = list(args)
    args2[12] = ctypes.c_void_p(0x10008)  # misaligned dS_final
    assert L.muir_chunk_bwd(ctypes.byref(shp), *args2, ctypes.c_size_t(0), None) == 1
    args3 = list(args)
    args3[10] = FAKE  # saved intermediates without the saved chunk states
    assert L.muir_chunk_bwd(ctypes.byref(shp), *args3, ctypes.c_size_t(0), None) == 1


def test_recurrent_step_rejects_bad_arguments(L):
    P = [FAKE] * 6
    assert L.muir_recurrent_step(0, 16, 128, 128, 0, 1, *P, None, 0, FAKE, FAKE, None) == 1
    assert L.muir_recurrent_step(2, 16, 96, 96, 0, 1, *P, None, 0, FAKE, FAKE, None) == 2
    assert L.muir_recurrent_step(2, 16, 128, 128, 0, 1, *P, None, 2, FAKE, FAKE, None) == 1
    assert L.muir_recurrent_step(2, 16, 128, 128, 0, 1, *P, None, 0, None, FAKE, None) == 1
    assert L.muir_recurrent_step(2, 16, 128, 128, 3, 1, *P, None, 0, FAKE, FAKE, None) == 1


def _cu(vals):
    return (ctypes.c_longlong * len(vals))(*vals)


def test_varlen_rejects_bad_offsets(L):
    import gated_delta_rule_115_b200 as m
    shp = _shape(m, T=100)
    fwd = lambda s, n, cu, **kw: L.muir_chunk_fwd_varlen(  # noqa: E731
        ctypes.byref(s), n, cu, *([FAKE] * 7), None, FAKE, None, kw.get("ws"),
        ctypes.c_size_t(kw.get("ws_bytes", 0)), None)
    # every case is rejected on the host before anything is enqueued
    assert fwd(_shape(m, B=2, T=100), 2, _cu([0, 40, 100])) == 1   # B must be 1
    assert fwd(shp, 2, _cu([1, 40, 100])) == 1                     # cu[0] != 0
    assert fwd(shp, 2, _cu([0, 60, 40])) == 1                      # decreasing
    assert fwd(shp, 2, _cu([0, 40, 99])) == 1                      # last != T
    assert fwd(shp, 0, _cu([0])) == 1                              # no sequence
    assert fwd(shp, 2, None) == 1
    assert fwd(_shape(m, T=100, dk=96, dv=96), 2, _cu([0, 40, 100])) == 2
    assert fwd(shp, 2, _cu([0, 40, 100])) == 3                     # valid, needs workspace
    assert L.muir_chunk_varlen_workspace(ctypes.byref(shp), 2, _cu([0, 60, 40]), 0) == 0
    # the workspace is the largest single sequence's
    one = L.muir_chunk_fwd_workspace(ctypes.byref(_shape(m, T=60)))
    assert L.muir_chunk_varlen_workspace(ctypes.byref(shp), 2, _cu([0, 40, 100]), 0) == one
    oneb = L.muir_chunk_bwd_workspace(ctypes.byref(_shape(m, T=60)))
    assert L.muir_chunk_varlen_workspace(ctypes.byref(shp), 2, _cu([0, 40, 100]), 1) == oneb
    args = [FAKE] * 7 + [None, FAKE, None] + [FAKE] * 7 + [None, None]
    assert L.muir_chunk_bwd_varlen(ctypes.byref(shp), 2, _cu([0, 50, 49]), *args,
                                   ctypes.c_size_t(0), None) == 1


def test_qk_prologue_rejects_bad_arguments(L):
    # every case is rejected on the host before anything is enqueued
    assert L.muir_qk_prologue(0, 128, 0, None, None, None) == 0          # empty: no-op
    assert L.muir_qk_prologue(-1, 128, 0, FAKE, FAKE, None) == 1
    assert L.muir_qk_prologue(16, 96, 0, FAKE, FAKE, None) == 2          # head dim
    assert L.muir_qk_prologue(16, 128, 5, FAKE, FAKE, None) == 1         # dtype
    assert L.muir_qk_prologue(16, 128, 0, None, FAKE, None) == 1
    assert L.muir_qk_prologue(16, 128, 0, FAKE, ctypes.c_void_p(0x10008), None) == 1
    assert L.muir_qk_prologue_bwd(0, 64, 1, None, None, None, None) == 0
    assert L.muir_qk_prologue_bwd(16, 32, 1, FAKE, FAKE, FAKE, None) == 2
    assert L.muir_qk_prologue_bwd(16, 64, 1, FAKE, None, FAKE, None) == 1
    assert L.muir_qk_prologue_bwd(16, 64, 1, FAKE, FAKE, ctypes.c_void_p(0x10004), None) == 1


def test_binding_refuses_cpu_tensors(L):
    import torch
    import gated_delta_rule_115_b200 as m
    x = torch.zeros(1, 2, 64)
    with pytest.raises(ValueError):
        m.recurrent_step(x, x, x, x, x, x, None, torch.zeros(1, 2, 64, 64), out_dtype=torch.float32,
                         o=torch.zeros(1, 2, 64))


def test_fused_workspace_host_checks(L):
    """muir_chunk_fused_workspace: 0 where a fused stage cannot run (ragged T,
    fp32 inputs, head dim 64, chunk 64) or for a bad fusion; more than the
    plain workspace where it can; equal to it with both stages off."""
    import gated_delta_rule_115_b200 as m
    on = m.MuirFusion(None, 1)
    off = m.MuirFusion(None, 0)
    good = _shape(m, T=512, dk=128, dv=128, chunk=128)
    for backward in (0, 1):
        plain = (L.muir_chunk_bwd_workspace if backward else L.muir_chunk_fwd_workspace)(
            ctypes.byref(good))
        assert L.muir_chunk_fused_workspace(ctypes.byref(good), ctypes.byref(on), backward) > plain
        assert L.muir_chunk_fused_workspace(ctypes.byref(good), ctypes.byref(off), backward) == plain
    for bad in (_shape(m, T=500, dk=128, dv=128, chunk=128),
                _shape(m, T=512, dk=128, dv=128, chunk=128, in_dtype=1),
                _shape(m, T=512, chunk=128),
                _shape(m, T=512, dk=128, dv=128, chunk=64)):
        assert L.muir_chunk_fused_workspace(ctypes.byref(bad), ctypes.byref(on), 0) == 0
    assert L.muir_chunk_fused_workspace(ctypes.byref(good), ctypes.byref(m.MuirFusion(None, 2)), 0) == 0
    assert L.muir_chunk_fused_workspace(ctypes.byref(good), None, 0) == 0


def test_debug_build_compiles(tmp_path):
    """The MUIR_DEBUG variant of the C-ABI layer (pointer residency checks)
    compiles for sm_100a."""
    import subprocess
    src = os.path.join(ROOT, "gated_delta_rule_115_b200", "csrc", "api.cu")
    r = subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-std=c++17", "-Xcompiler", "-fPIC", "-DMUIR_DEBUG=1", "-c", src, "-o",
                        str(tmp_path / "api_debug.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_selftest_rejects_bad_limits(L):
    for bad in (0, -5, 1000001):
        assert L.muir_selftest_expired_wait(bad, None) == 1  # MUIR_ERR_INVALID_ARG
