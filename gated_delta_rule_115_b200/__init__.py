"""Python binding of libmuir, the Muir gated delta rule on one NVIDIA B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libmuir.so`` (built in-tree by ``gated_delta_rule_115_b200.build``)
behind the C ABI declared in ``include/muir.h``.  PyTorch supplies device
memory and the current CUDA stream.  There is no CPU fallback: if the library
is missing or a call fails, an exception is raised.

Recurrence (arXiv 2611.08376, wolonglab.org page, "Methodology", eq:gdn2 and
eq:ours), per batch and head, state S in R^{dk x dv} with rows = key channels:

    S_t = diag(exp g_t) S_{t-1} - (e_t*k_t)(k_t^T diag(exp g_t) S_{t-1}) + k_t (w_t*v_t)^T
    o_t = S_t^T (gamma_t * q_t)

Per-token tensors are ``[B, T, H, d]``; states ``[B, H, dk, dv]`` float32.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MuirError", "lib", "chunk_fwd", "chunk_bwd", "chunk_fwd_varlen", "chunk_bwd_varlen",
    "recurrent_step", "qk_prologue", "chunk_fwd_fused", "chunk_bwd_fused", "MuirFusion",
    "qk_prologue_bwd", "fwd_workspace_bytes", "bwd_workspace_bytes", "MuirChunkFunction",
    "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuir.so")

MUIR_BF16, MUIR_FP32 = 0, 1
_STATUS = {0: "MUIR_OK", 1: "MUIR_ERR_INVALID_ARG", 2: "MUIR_ERR_UNSUPPORTED",
           3: "MUIR_ERR_WORKSPACE", 4: "MUIR_ERR_CUDA", 5: "MUIR_ERR_DEVICE_TIMEOUT"}


class MuirError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        msg = _lib.muir_status_string(code).decode() if _lib is not None else _STATUS.get(code)
        super().__init__(f"{fn} failed: {msg}")


class MuirShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


class MuirGateFamily(ctypes.Structure):
    _fields_ = [("off", ctypes.c_int), ("rank", ctypes.c_int), ("U", ctypes.c_void_p),
                ("bias", ctypes.c_void_p)]


class MuirFusion(ctypes.Structure):
    _fields_ = [("z_out", ctypes.c_void_p), ("qk_raw", ctypes.c_int),
                ("latent", ctypes.c_void_p), ("R", ctypes.c_int), ("fam", MuirGateFamily * 5)]


class MuirFusionGrads(ctypes.Structure):
    _fields_ = [("dlatent", ctypes.c_void_p), ("dU", ctypes.c_void_p * 5),
                ("dbias", ctypes.c_void_p * 5)]


# gate families of the fused projection, in the latent's column order
GATE_FAMILIES = ("f", "b", "g", "w", "q")


_lib = None


def lib():
    """The loaded ``libmuir.so`` (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m gated_delta_rule_115_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        SP = ctypes.POINTER(MuirShape)
        L.muir_selftest_expired_wait.argtypes = [I, P]
        L.muir_selftest_expired_wait.restype = I
        L.muir_device_wait_status.argtypes = []
        L.muir_device_wait_status.restype = I
        L.muir_status_string.argtypes = [I]
        L.muir_status_string.restype = ctypes.c_char_p
        L.muir_chunk_aux_floats.argtypes = [SP]
        L.muir_chunk_aux_floats.restype = ctypes.c_size_t
        L.muir_chunk_fwd_workspace.argtypes = [SP]
        L.muir_chunk_fwd_workspace.restype = S
        L.muir_chunk_bwd_workspace.argtypes = [SP]
        L.muir_chunk_bwd_workspace.restype = S
        L.muir_chunk_fwd.argtypes = [SP] + [P] * 14 + [S, P]
        L.muir_chunk_fwd.restype = I
        L.muir_chunk_bwd.argtypes = [SP] + [P] * 22 + [S, P]
        L.muir_chunk_bwd.restype = I
        L.muir_recurrent_step.argtypes = [I, I, I, I, I, I] + [P] * 7 + [I, P, P, P]
        L.muir_recurrent_step.restype = I
        LLP = ctypes.POINTER(ctypes.c_longlong)
        L.muir_chunk_varlen_workspace.argtypes = [SP, I, LLP, I]
        L.muir_chunk_varlen_workspace.restype = S
        L.muir_chunk_fwd_varlen.argtypes = [SP, I, LLP] + [P] * 11 + [S, P]
        L.muir_chunk_fwd_varlen.restype = I
        L.muir_chunk_bwd_varlen.argtypes = [SP, I, LLP] + [P] * 19 + [S, P]
        L.muir_chunk_bwd_varlen.restype = I
        L.muir_qk_prologue.argtypes = [ctypes.c_longlong, I, I, P, P, P]
        L.muir_qk_prologue.restype = I
        L.muir_qk_prologue_bwd.argtypes = [ctypes.c_longlong, I, I, P, P, P, P]
        L.muir_qk_prologue_bwd.restype = I
        FP = ctypes.POINTER(MuirFusion)
        L.muir_chunk_fused_workspace.argtypes = [SP, FP, I]
        L.muir_chunk_fused_workspace.restype = S
        L.muir_chunk_fwd_fused.argtypes = [SP, FP] + [P] * 15 + [S, P]
        L.muir_chunk_fwd_fused.restype = I
        L.muir_chunk_bwd_fused.argtypes = [SP, FP] + [P] * 25 + [S, P]
        L.muir_chunk_bwd_fused.restype = I
        L.muir_chunk_fwd_noalloc.argtypes = [SP] + [P] * 10 + [P]
        L.muir_chunk_fwd_noalloc.restype = I
        L.muir_profile_enable.argtypes = [I]
        L.muir_profile_enable.restype = None
        L.muir_profile_reset.argtypes = []
        L.muir_profile_reset.restype = None
        L.muir_profile_collect.argtypes = []
        L.muir_profile_collect.restype = I
        L.muir_profile_count.argtypes = []
        L.muir_profile_count.restype = I
        L.muir_profile_name.argtypes = [I]
        L.muir_profile_name.restype = ctypes.c_char_p
        L.muir_profile_total_ms.argtypes = [I]
        L.muir_profile_total_ms.restype = ctypes.c_double
        L.muir_profile_launches.argtypes = [I]
        L.muir_profile_launches.restype = ctypes.c_longlong
        _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MUIR_BF16
    if t.dtype == torch.float32:
        return MUIR_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmuir takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libmuir takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise MuirError(fn, rc)


def _shape(q, v, chunk, out_dtype):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    od = _dt(q) if out_dtype is None else (MUIR_BF16 if out_dtype == torch.bfloat16 else MUIR_FP32)
    return MuirShape(B, T, H, dk, dv, chunk, _dt(q), od)


def device_wait_status() -> None:
    """Synchronise the device and raise MuirError if a bounded wait inside a
    chunk kernel expired since the previous check (muir_device_wait_status)."""
    _check("muir_device_wait_status", lib().muir_device_wait_status())


def fwd_workspace_bytes(B, T, H, d, chunk, dtype=torch.bfloat16) -> int:
    s = MuirShape(B, T, H, d, d, chunk, MUIR_BF16 if dtype == torch.bfloat16 else MUIR_FP32, 0)
    return int(lib().muir_chunk_fwd_workspace(ctypes.byref(s)))


def bwd_workspace_bytes(B, T, H, d, chunk, dtype=torch.bfloat16) -> int:
    s = MuirShape(B, T, H, d, d, chunk, MUIR_BF16 if dtype == torch.bfloat16 else MUIR_FP32, 0)
    return int(lib().muir_chunk_bwd_workspace(ctypes.byref(s)))


def _workspace(nbytes, dev, ws):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=dev)


def chunk_fwd(q, k, v, g, e, w, gamma, S0=None, chunk=64, out_dtype=None,
              return_chunk_states=False, return_saved=False, save_aux=False, ws=None):
    """Chunkwise forward.  Returns ``(o, S_final)``; with ``return_chunk_states``
    ``(o, S_final, S_chunks)`` where ``S_chunks[b,h,n]`` is the state at the start
    of chunk ``n``; with ``return_saved`` ``(o, S_final, S_chunks, M_chunks)``
    where ``M_chunks[b,h,n]`` is chunk n's transition, and with ``save_aux`` as
    well a fifth element ``aux``, the per-chunk intermediates
    (``muir_chunk_aux_floats``).  All are reusable by :func:`chunk_bwd`."""
    L = lib()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    shp = _shape(q, v, chunk, out_dtype)
    od = torch.bfloat16 if shp.out_dtype == MUIR_BF16 else torch.float32
    o = torch.empty(B, T, H, dv, dtype=od, device=q.device)
    S_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    Sc = (torch.empty(B, H, -(-T // chunk), dk, dv, dtype=torch.float32, device=q.device)
          if (return_chunk_states or return_saved) else None)
    Mc = (torch.empty(B, H, -(-T // chunk), dk, dk, dtype=torch.float32, device=q.device)
          if return_saved else None)
    aux = None
    if return_saved and save_aux:
        aux = torch.empty(int(L.muir_chunk_aux_floats(ctypes.byref(shp))), dtype=torch.float32,
                          device=q.device)
    need = int(L.muir_chunk_fwd_workspace(ctypes.byref(shp)))
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_fwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(e),
                          _ptr(w), _ptr(gamma), _ptr(S0), _ptr(o), _ptr(S_final), _ptr(Sc),
                          _ptr(Mc), _ptr(aux), _ptr(wsb),
                          ctypes.c_size_t(0 if wsb is None else wsb.numel()), _stream(q.device))
    _check("muir_chunk_fwd", rc)
    if return_saved:
        return (o, S_final, Sc, Mc, aux) if save_aux else (o, S_final, Sc, Mc)
    return (o, S_final, Sc) if return_chunk_states else (o, S_final)


def chunk_bwd(q, k, v, g, e, w, gamma, S0, dO, dS_final=None, chunk=64, S_chunks=None,
              M_chunks=None, aux=None, ws=None):
    """Gradients of ``sum(o*dO) + sum(S_final*dS_final)``.  Returns a dict with
    ``dq, dk, dv, dg, de, dw, dgamma`` (input dtype) and ``dS0`` (float32).
    ``S_chunks`` / ``M_chunks`` / ``aux`` from :func:`chunk_fwd` skip
    recomputation (``aux`` only together with ``S_chunks``)."""
    L = lib()
    shp = _shape(q, v, chunk, None)
    grads = {n: torch.empty_like(x) for n, x in
             dict(dq=q, dk=k, dv=v, dg=g, de=e, dw=w, dgamma=gamma).items()}
    B, T, H, dk = q.shape
    grads["dS0"] = torch.empty(B, H, dk, v.shape[-1], dtype=torch.float32, device=q.device)
    need = int(L.muir_chunk_bwd_workspace(ctypes.byref(shp)))
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_bwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(e),
                          _ptr(w), _ptr(gamma), _ptr(S0), _ptr(S_chunks), _ptr(M_chunks), _ptr(aux),
                          _ptr(dO),
                          _ptr(dS_final), _ptr(grads["dq"]), _ptr(grads["dk"]),
                          _ptr(grads["dv"]), _ptr(grads["dg"]), _ptr(grads["de"]),
                          _ptr(grads["dw"]), _ptr(grads["dgamma"]), _ptr(grads["dS0"]),
                          _ptr(wsb), ctypes.c_size_t(0 if wsb is None else wsb.numel()),
                          _stream(q.device))
    _check("muir_chunk_bwd", rc)
    return grads


def _fusion(z_out, qk_raw, latent=None, proj=None):
    """``proj`` maps a family name (``GATE_FAMILIES``) to ``(offset, U, bias)``:
    U [rank, H*dk] bf16, bias [H*dk] float32."""
    f = MuirFusion()
    f.z_out = None if z_out is None else _ptr(z_out).value
    f.qk_raw = int(bool(qk_raw))
    if latent is not None:
        f.latent = _ptr(latent).value
        f.R = latent.shape[-1]
        for name, (off, U, bias) in (proj or {}).items():
            fam = f.fam[GATE_FAMILIES.index(name)]
            fam.off, fam.rank = int(off), U.shape[0]
            fam.U, fam.bias = _ptr(U).value, _ptr(bias).value
    return f


def chunk_fwd_fused(q, k, v, g, e, w, gamma, S0=None, z_out=None, qk_raw=False, chunk=128,
                    out_dtype=None, save=True, ws=None, latent=None, proj=None):
    """Forward with the fused stages (``muir_chunk_fwd_fused``): ``qk_raw``
    means q and k are the raw pre-activations (SiLU and the unit L2 norm are
    applied in the kernels); ``z_out`` is the output gate's pre-activation
    (the output is ``o * sigmoid(z_out)``); ``latent`` [B, T, R] with ``proj``
    (family -> (offset, U, bias)) projects those families' gates from the
    latent (their tensor arguments may be None).  Returns ``(o, S_final, saved)``;
    ``saved`` (None unless ``save``) holds what :func:`chunk_bwd_fused` reuses:
    ``S_chunks``, ``M_chunks``, ``aux`` and, with a gate, ``o_pre``."""
    L = lib()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    shp = _shape(q, v, chunk, out_dtype)
    fu = _fusion(z_out, qk_raw, latent, proj)
    od = torch.bfloat16 if shp.out_dtype == MUIR_BF16 else torch.float32
    o = torch.empty(B, T, H, dv, dtype=od, device=q.device)
    gated = z_out is not None or (proj is not None and "g" in proj)
    o_pre = torch.empty_like(o) if gated else None
    S_final = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    Sc = Mc = aux = None
    if save:
        n = -(-T // chunk)
        Sc = torch.empty(B, H, n, dk, dv, dtype=torch.float32, device=q.device)
        Mc = torch.empty(B, H, n, dk, dk, dtype=torch.float32, device=q.device)
        aux = torch.empty(int(L.muir_chunk_aux_floats(ctypes.byref(shp))), dtype=torch.float32,
                          device=q.device)
    need = int(L.muir_chunk_fused_workspace(ctypes.byref(shp), ctypes.byref(fu), 0))
    if need == 0:
        raise MuirError("muir_chunk_fused_workspace", 2)
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_fwd_fused(ctypes.byref(shp), ctypes.byref(fu), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(e), _ptr(w), _ptr(gamma), _ptr(S0), _ptr(o),
                                _ptr(o_pre), _ptr(S_final), _ptr(Sc), _ptr(Mc), _ptr(aux),
                                _ptr(wsb), ctypes.c_size_t(wsb.numel()), _stream(q.device))
    _check("muir_chunk_fwd_fused", rc)
    saved = dict(S_chunks=Sc, M_chunks=Mc, aux=aux, o_pre=o_pre) if save else None
    return o, S_final, saved


def chunk_bwd_fused(q, k, v, g, e, w, gamma, S0, dO, dS_final=None, z_out=None, qk_raw=False,
                    o_pre=None, saved=None, chunk=128, ws=None, latent=None, proj=None):
    """Gradients through :func:`chunk_fwd_fused` (``muir_chunk_bwd_fused``):
    ``dO`` is the gradient of the (gated) output.  Returns the dict of
    :func:`chunk_bwd` plus ``dz_out`` with a gate; dq and dk are with respect
    to the raw q and k when ``qk_raw``.  ``saved`` from the forward skips
    recomputation; with a gate, ``o_pre`` (or ``saved["o_pre"]``) is required."""
    L = lib()
    shp = _shape(q, v, chunk, None)
    if saved is not None and o_pre is None:
        o_pre = saved.get("o_pre")
    if o_pre is not None:
        shp.out_dtype = MUIR_BF16 if o_pre.dtype == torch.bfloat16 else MUIR_FP32
    fu = _fusion(z_out, qk_raw, latent, proj)
    grads = {n: (torch.empty_like(x) if x is not None else None) for n, x in
             dict(dq=q, dk=k, dv=v, dg=g, de=e, dw=w, dgamma=gamma).items()}
    B, T, H, dk = q.shape
    grads["dS0"] = torch.empty(B, H, dk, v.shape[-1], dtype=torch.float32, device=q.device)
    dz = torch.empty_like(z_out) if z_out is not None else None
    fg = None
    if latent is not None:
        fg = MuirFusionGrads()
        grads["dlatent"] = torch.empty_like(latent)
        fg.dlatent = _ptr(grads["dlatent"]).value
        for name, (off, U, bias) in proj.items():
            i = GATE_FAMILIES.index(name)
            grads["dU_" + name] = torch.empty(U.shape, dtype=torch.float32, device=q.device)
            grads["dbias_" + name] = torch.empty(bias.shape, dtype=torch.float32, device=q.device)
            fg.dU[i] = _ptr(grads["dU_" + name]).value
            fg.dbias[i] = _ptr(grads["dbias_" + name]).value
    Sc, Mc, aux = ((saved["S_chunks"], saved["M_chunks"], saved["aux"]) if saved is not None
                   else (None, None, None))
    need = int(L.muir_chunk_fused_workspace(ctypes.byref(shp), ctypes.byref(fu), 1))
    if need == 0:
        raise MuirError("muir_chunk_fused_workspace", 2)
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_bwd_fused(ctypes.byref(shp), ctypes.byref(fu), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(e), _ptr(w), _ptr(gamma), _ptr(S0), _ptr(Sc),
                                _ptr(Mc), _ptr(aux), _ptr(o_pre), _ptr(dO), _ptr(dS_final),
                                *[_ptr(grads[n]) for n in ("dq", "dk", "dv", "dg", "de", "dw",
                                                           "dgamma")],
                                _ptr(dz), _ptr(grads["dS0"]),
                                ctypes.byref(fg) if fg is not None else None, _ptr(wsb),
                                ctypes.c_size_t(wsb.numel()), _stream(q.device))
    _check("muir_chunk_bwd_fused", rc)
    for n in ("dg", "de", "dw", "dgamma"):
        if grads[n] is None:
            del grads[n]
    if dz is not None:
        grads["dz_out"] = dz
    return grads


def recurrent_step(q, k, v, g, e, w, gamma, S, gamma_static=False, out_dtype=None, o=None):
    """One decode token for every (b, h); ``S`` ([B,H,dk,dv] float32) is
    updated in place.  ``gamma`` is ``[B,H,dk]``, ``[H,dk]`` with
    ``gamma_static=True``, or None.  Returns ``o`` ([B,H,dv])."""
    L = lib()
    B, H, dk = q.shape
    dv = v.shape[-1]
    od = q.dtype if out_dtype is None else out_dtype
    if o is None:
        o = torch.empty(B, H, dv, dtype=od, device=q.device)
    rc = L.muir_recurrent_step(B, H, dk, dv, _dt(q), _dt(o), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(g), _ptr(e), _ptr(w), _ptr(gamma), int(bool(gamma_static)),
                               _ptr(S), _ptr(o), _stream(q.device))
    _check("muir_recurrent_step", rc)
    return o


def _cu(cu_seqlens):
    vals = [int(c) for c in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return len(vals) - 1, (ctypes.c_longlong * len(vals))(*vals)


def chunk_fwd_varlen(q, k, v, g, e, w, gamma, cu_seqlens, S0=None, chunk=64, out_dtype=None,
                     ws=None):
    """Forward over packed sequences: per-token tensors ``[1, T, H, d]`` with
    sequence i at rows ``cu_seqlens[i]:cu_seqlens[i+1]`` (a host list or CPU
    tensor).  ``S0`` is ``[num_seqs, H, dk, dv]`` or None.  Returns
    ``(o, S_final)`` with ``S_final`` of shape ``[num_seqs, H, dk, dv]``."""
    L = lib()
    n, cu = _cu(cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    shp = _shape(q, v, chunk, out_dtype)
    od = torch.bfloat16 if shp.out_dtype == MUIR_BF16 else torch.float32
    o = torch.empty(B, T, H, dv, dtype=od, device=q.device)
    S_final = torch.empty(n, H, dk, dv, dtype=torch.float32, device=q.device)
    need = int(L.muir_chunk_varlen_workspace(ctypes.byref(shp), n, cu, 0))
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_fwd_varlen(ctypes.byref(shp), n, cu, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(e), _ptr(w), _ptr(gamma), _ptr(S0), _ptr(o), _ptr(S_final),
                                 _ptr(wsb), ctypes.c_size_t(0 if wsb is None else wsb.numel()),
                                 _stream(q.device))
    _check("muir_chunk_fwd_varlen", rc)
    return o, S_final


def chunk_bwd_varlen(q, k, v, g, e, w, gamma, cu_seqlens, S0, dO, dS_final=None, chunk=64,
                     ws=None):
    """Gradients of ``sum(o*dO) + sum(S_final*dS_final)`` over packed sequences
    (see :func:`chunk_fwd_varlen`); returns the dict of :func:`chunk_bwd` with
    ``dS0`` of shape ``[num_seqs, H, dk, dv]``."""
    L = lib()
    n, cu = _cu(cu_seqlens)
    shp = _shape(q, v, chunk, None)
    grads = {nm: torch.empty_like(x) for nm, x in
             dict(dq=q, dk=k, dv=v, dg=g, de=e, dw=w, dgamma=gamma).items()}
    _, _, H, dk = q.shape
    grads["dS0"] = torch.empty(n, H, dk, v.shape[-1], dtype=torch.float32, device=q.device)
    need = int(L.muir_chunk_varlen_workspace(ctypes.byref(shp), n, cu, 1))
    wsb = _workspace(need, q.device, ws)
    rc = L.muir_chunk_bwd_varlen(ctypes.byref(shp), n, cu, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(e), _ptr(w), _ptr(gamma), _ptr(S0), _ptr(dO),
                                 _ptr(dS_final), *[_ptr(grads[nm]) for nm in
                                                   ("dq", "dk", "dv", "dg", "de", "dw", "dgamma")],
                                 _ptr(grads["dS0"]), _ptr(wsb),
                                 ctypes.c_size_t(0 if wsb is None else wsb.numel()),
                                 _stream(q.device))
    _check("muir_chunk_bwd_varlen", rc)
    return grads


def qk_prologue(x, out=None):
    """``SiLU(x) / max(||SiLU(x)||, 1e-12)`` over the last dim (64 or 128) of a
    contiguous bf16/float32 tensor; ``out`` may be ``x`` (in place)."""
    L = lib()
    if out is None:
        out = torch.empty_like(x)
    d = x.shape[-1]
    rc = L.muir_qk_prologue(x.numel() // d, d, _dt(x), _ptr(x), _ptr(out), _stream(x.device))
    _check("muir_qk_prologue", rc)
    return out


def qk_prologue_bwd(x, dy, out=None):
    """Gradient of :func:`qk_prologue` with respect to ``x`` for upstream ``dy``."""
    L = lib()
    if out is None:
        out = torch.empty_like(x)
    d = x.shape[-1]
    rc = L.muir_qk_prologue_bwd(x.numel() // d, d, _dt(x), _ptr(x), _ptr(dy), _ptr(out),
                                _stream(x.device))
    _check("muir_qk_prologue_bwd", rc)
    return out


class MuirChunkFunction(torch.autograd.Function):
    """Autograd wrapper: forward saves the chunk states, backward reuses them."""

    @staticmethod
    def forward(ctx, q, k, v, g, e, w, gamma, S0, chunk):
        o, S_final, Sc, Mc, aux = chunk_fwd(q, k, v, g, e, w, gamma, S0, chunk=chunk,
                                            return_saved=True, save_aux=True)
        ctx.save_for_backward(q, k, v, g, e, w, gamma, S0, Sc, Mc, aux)
        ctx.chunk = chunk
        return o, S_final

    @staticmethod
    def backward(ctx, dO, dS_final):
        q, k, v, g, e, w, gamma, S0, Sc, Mc, aux = ctx.saved_tensors
        gr = chunk_bwd(q, k, v, g, e, w, gamma, S0, dO.contiguous().to(q.dtype),
                       None if dS_final is None else dS_final.contiguous().float(),
                       chunk=ctx.chunk, S_chunks=Sc, M_chunks=Mc, aux=aux)
        return (gr["dq"], gr["dk"], gr["dv"], gr["dg"], gr["de"], gr["dw"], gr["dgamma"],
                gr["dS0"] if S0 is not None else None, None)
