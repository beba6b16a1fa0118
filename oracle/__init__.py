"""fp64 CPU oracle of the Muir gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The CUDA library never calls it, and
nothing here imports the CUDA library: the two share no code.

Two independent C sources are wrapped:

* ``muir_ref.c`` -- the token-by-token recurrence of "Muir: Linear Attention
  with Sensitivity-Allocated Gating and Matched-Filter Readout" (arXiv
  2611.08376; wolonglab.org page, "Methodology", eq:gdn2 and eq:ours), its
  back-propagation through time, and the single-token decode step.
* ``muir_chunk_ref.c`` -- the chunked (WY / UT) form of the same recurrence,
  derived by unrolling it over a chunk (same page, "Methodology": each chunk is
  a triangular system), with exact exponent differences.

and, in numpy below, the q/k feature prologue (SiLU, then unit L2 norm per
token-head row; same page, "Methodology" and fig. 3(b)) with its gradient, the
output gate o * sigmoid(z) with its gradient, the fused layer composed of the
three (``fwd_fused`` / ``bwd_fused``), and the fused low-rank gate projection
(one latent per token, five up-projections with channel biases, eq:ours_proj)
with its gradient.

Every function takes numpy-convertible arrays, computes in float64 and returns
float64 numpy arrays.  Per-token tensors are ``[B, T, H, d]``; states are
``[B, H, dk, dv]``.

Pins (what fixes these functions other than themselves) live in
``tests/test_oracle_pins.py``, ``tests/test_qk_oracle.py`` (the prologue) and
``tests/test_fused_oracle.py`` (output gate, fused composition),
``tests/test_gate_oracle.py`` (gate projection):
linear-attention and gated-linear-attention
closed forms, the delta rule (Widrow-Hoff), an exact-retrieval invariant,
pure decay, chunk-size invariance, linearity, column equivariance, state
passing, decode/recurrence equivalence, a hand-computed example in
``tests/golden/``, central finite differences and torch autograd for the
gradients.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_SOURCES = ["muir_ref.c", "muir_chunk_ref.c"]
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, no fast-math)."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if not force and os.path.exists(_LIB_PATH):
        newest = max(os.path.getmtime(s) for s in srcs)
        if os.path.getmtime(_LIB_PATH) >= newest:
            return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
           "-pthread", "-o", tmp] + srcs + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.muir_ref_fwd.argtypes = [I] * 5 + [P] * 10 + [I]
        lib.muir_ref_bwd.argtypes = [I] * 5 + [P] * 18 + [I, I]
        lib.muir_ref_step.argtypes = [I] * 4 + [P] * 7 + [I, P, P]
        lib.muir_chunk_ref_fwd.argtypes = [I] * 6 + [P] * 11 + [I]
        for f in (lib.muir_ref_fwd, lib.muir_ref_bwd, lib.muir_ref_step,
                  lib.muir_chunk_ref_fwd):
            f.restype = I
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _dims(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    return B, T, H, dk, dv


def fwd(q, k, v, g, e, w, gamma=None, S0=None, threads=None):
    """Token-by-token forward.  Returns ``(o [B,T,H,dv], S_T [B,H,dk,dv])``."""
    lib = _load()
    q, k, v, g, e, w, gamma, S0 = map(_f64, (q, k, v, g, e, w, gamma, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.zeros((B, T, H, dv))
    S = np.zeros((B, H, dk, dv))
    rc = lib.muir_ref_fwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(e), _p(w),
                          _p(gamma), _p(S0), _p(o), _p(S), threads or default_threads())
    if rc:
        raise ValueError("muir_ref_fwd: bad shape")
    return o, S


def bwd(q, k, v, g, e, w, gamma=None, S0=None, dO=None, dS_final=None, ckpt=64,
        threads=None):
    """Back-propagation through time of ``sum(o*dO) + sum(S_T*dS_final)``.

    Returns a dict with ``dq, dk, dv, dg, de, dw, dgamma`` ([B,T,H,d]) and
    ``dS0`` ([B,H,dk,dv]).
    """
    lib = _load()
    q, k, v, g, e, w, gamma, S0, dO, dS_final = map(
        _f64, (q, k, v, g, e, w, gamma, S0, dO, dS_final))
    B, T, H, dk, dv = _dims(q, v)
    if dO is None:
        dO = np.zeros((B, T, H, dv))
    out = {n: np.zeros((B, T, H, dk)) for n in ("dq", "dk", "dg", "de", "dgamma")}
    out.update({n: np.zeros((B, T, H, dv)) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    rc = lib.muir_ref_bwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(e), _p(w),
                          _p(gamma), _p(S0), _p(dO), _p(dS_final), _p(out["dq"]),
                          _p(out["dk"]), _p(out["dv"]), _p(out["dg"]), _p(out["de"]),
                          _p(out["dw"]), _p(out["dgamma"]), _p(out["dS0"]), int(ckpt),
                          threads or default_threads())
    if rc:
        raise ValueError("muir_ref_bwd: bad shape")
    return out


def chunk_fwd(q, k, v, g, e, w, gamma=None, S0=None, chunk=64, threads=None):
    """Chunked (WY form) forward.  Returns ``(o, S_T, S_chunks)`` where
    ``S_chunks[b, h, n]`` is the state at the start of chunk ``n``."""
    lib = _load()
    q, k, v, g, e, w, gamma, S0 = map(_f64, (q, k, v, g, e, w, gamma, S0))
    B, T, H, dk, dv = _dims(q, v)
    n = (T + chunk - 1) // chunk
    o = np.zeros((B, T, H, dv))
    S = np.zeros((B, H, dk, dv))
    Sc = np.zeros((B, H, n, dk, dv))
    rc = lib.muir_chunk_ref_fwd(B, T, H, dk, dv, int(chunk), _p(q), _p(k), _p(v), _p(g),
                                _p(e), _p(w), _p(gamma), _p(S0), _p(o), _p(S), _p(Sc),
                                threads or default_threads())
    if rc:
        raise ValueError("muir_chunk_ref_fwd: bad shape")
    return o, S, Sc


def step(q, k, v, g, e, w, gamma, S, gamma_static=False):
    """One decode token for every (b, h).  Per-token inputs are ``[B, H, d]``;
    ``gamma`` is ``[B, H, dk]``, or ``[H, dk]`` with ``gamma_static=True``, or
    None.  Returns ``(o [B,H,dv], S_new)``; the input ``S`` is not modified."""
    lib = _load()
    q, k, v, g, e, w, gamma = map(_f64, (q, k, v, g, e, w, gamma))
    S = _f64(S).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((B, H, dv))
    rc = lib.muir_ref_step(B, H, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(e), _p(w),
                           _p(gamma), int(bool(gamma_static)), _p(S), _p(o))
    if rc:
        raise ValueError("muir_ref_step: bad shape")
    return o, S


# ------------------------------------------------------------ q/k prologue

QK_NORM_EPS = 1e-12  # guard of the norm: an all-zero row maps to zero


def qk_prologue(x):
    """``y = s / max(||s||, eps)`` with ``s = SiLU(x) = x * sigmoid(x)`` over the
    last axis (one token-head row of d channels), in float64.  The pages end
    the query and key pathways in SiLU and keep the key unit-normalised
    ("Methodology", fig. 3(b)); eps only guards the zero row."""
    x = _f64(x)
    s = x / (1.0 + np.exp(-x))
    n = np.maximum(np.sqrt((s * s).sum(axis=-1, keepdims=True)), QK_NORM_EPS)
    return s / n


def qk_prologue_bwd(x, dy):
    """Gradient of ``sum(dy * qk_prologue(x))`` with respect to x, in float64:
    the Jacobian of s -> s / ||s|| is (I - y y^T) / ||s|| (1 / eps times the
    identity below the guard), and SiLU'(x) = sig(x) (1 + x (1 - sig(x)))."""
    x, dy = _f64(x), _f64(dy)
    sig = 1.0 / (1.0 + np.exp(-x))
    s = x * sig
    nrm = np.sqrt((s * s).sum(axis=-1, keepdims=True))
    tiny = nrm < QK_NORM_EPS
    n = np.maximum(nrm, QK_NORM_EPS)
    y = s / n
    ds = (dy - np.where(tiny, 0.0, y * (y * dy).sum(axis=-1, keepdims=True))) / n
    return ds * sig * (1.0 + x * (1.0 - sig))


# ------------------------------------------------------------ output gate

def out_gate(o, z):
    """Output gate applied after the mixer: ``o * sigmoid(z)``, elementwise, in
    float64.  The pages name a rank-128 gate g_t among the five gate families
    ("Methodology", fig. 3(b)-(c): ranks (r_f, r_b, r_g, r_w, r_q)); the tab:abl
    caption compares against a widened output gate, which identifies g_t as the
    output gate.  z is its pre-activation per token, head and value channel."""
    o, z = _f64(o), _f64(z)
    return o / (1.0 + np.exp(-z))


def out_gate_bwd(o, z, dy):
    """Gradients of ``sum(dy * out_gate(o, z))``: ``(do, dz)`` with
    ``do = dy sig(z)`` and ``dz = dy o sig(z) (1 - sig(z))``."""
    o, z, dy = _f64(o), _f64(z), _f64(dy)
    sig = 1.0 / (1.0 + np.exp(-z))
    return dy * sig, dy * o * sig * (1.0 - sig)


# ------------------------------------------------------------ fused layer

def fwd_fused(q, k, v, g, e, w, gamma=None, S0=None, z_out=None, qk_raw=False, threads=None):
    """The mixer with its optional fused stages, composed from the functions
    above in the order the pages' block applies them (fig. 3(b)): the q/k
    prologue on raw q and k (``qk_raw``), the recurrence, then the output gate
    on o (``z_out``).  Returns ``(o_gated, S_T, o)``: o is the pre-gate output
    (equal to o_gated without a gate)."""
    if qk_raw:
        q, k = qk_prologue(q), qk_prologue(k)
    o, S = fwd(q, k, v, g, e, w, gamma, S0, threads=threads)
    og = out_gate(o, z_out) if z_out is not None else o
    return og, S, o


def bwd_fused(q, k, v, g, e, w, gamma=None, S0=None, dO=None, dS_final=None, z_out=None,
              qk_raw=False, threads=None):
    """Gradients of ``sum(o_gated * dO) + sum(S_T * dS_final)`` through
    ``fwd_fused`` by the chain rule: the output gate's gradient, then the
    recurrence's back-propagation through time, then the prologue's Jacobian
    on dq and dk (gradients with respect to the raw q and k when ``qk_raw``).
    Returns the dict of ``bwd`` plus ``dz_out`` when a gate is given."""
    qh, kh = (qk_prologue(q), qk_prologue(k)) if qk_raw else (q, k)
    out = {}
    if z_out is not None:
        o, _ = fwd(qh, kh, v, g, e, w, gamma, S0, threads=threads)
        dO, out["dz_out"] = out_gate_bwd(o, z_out, dO)
    out.update(bwd(qh, kh, v, g, e, w, gamma, S0, dO=dO, dS_final=dS_final, threads=threads))
    if qk_raw:
        out["dq"] = qk_prologue_bwd(q, out["dq"])
        out["dk"] = qk_prologue_bwd(k, out["dk"])
    return out


# ------------------------------------------------------------ gate projection

# The five gate families of the fused low-rank projection ("Methodology";
# fig. 3(c): ranks (r_f, r_b, r_g, r_w, r_q) = (64, 64, 128, 128, 128), R_tot =
# 512), in the order their latent columns are laid out, with what each yields:
# f -> log decay g, b -> erase e, g -> the output gate's pre-activation z_out,
# w -> write w, q -> readout gain gamma.
GATE_FAMILIES = ("f", "b", "g", "w", "q")
GATE_OUTPUT = {"f": "g", "b": "e", "g": "z_out", "w": "w", "q": "gamma"}


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.logaddexp(0.0, x)


def _gate_act(fam, pre):
    """g = -softplus(pre) (log decay, <= 0); e, w, gamma = sigmoid(pre); the
    output gate's pre-activation passes through (its sigmoid is applied after
    the mixer)."""
    if fam == "f":
        return -_softplus(pre)
    if fam == "g":
        return pre
    return _sig(pre)


def _gate_act_grad(fam, pre):
    if fam == "f":
        return -_sig(pre)
    if fam == "g":
        return np.ones_like(pre)
    s = _sig(pre)
    return s * (1.0 - s)


def round_bf16(x):
    """Round to bfloat16 the way the kernels store a float32 value: first to
    float32 (the precision the kernels compute in), then to the nearest bf16,
    ties to even.  Returns float64 holding the bf16 values."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def gate_pre(lat, ups, H):
    """Pre-activations of the fused projection.  ``lat`` [B, T, R] is the
    per-token latent (shared by all heads); ``ups`` maps a family to
    ``(offset, U [r, H*d], bias [H*d])``: the family's latent columns are
    ``offset .. offset + r``.  Returns ``{family: pre [B, T, H, d]}``."""
    lat = _f64(lat)
    B, T, _ = lat.shape
    out = {}
    for fam, (off, U, bias) in ups.items():
        U, bias = _f64(U), _f64(bias)
        r = U.shape[0]
        pre = lat[:, :, off:off + r] @ U + bias
        out[fam] = pre.reshape(B, T, H, -1)
    return out


def gate_projection(lat, ups, H, rounded=True):
    """The gates the fused projection yields (``GATE_OUTPUT`` names), each
    [B, T, H, d]: activation of ``gate_pre``, rounded to bf16 when
    ``rounded`` (the gate dtype the kernels consume)."""
    pre = gate_pre(lat, ups, H)
    out = {}
    for fam, p in pre.items():
        a = _gate_act(fam, p)
        out[GATE_OUTPUT[fam]] = round_bf16(a) if rounded else a
    return out


def gate_projection_bwd(lat, ups, H, dgates):
    """Gradients of ``sum_X dgates[X] * gate_X`` through ``gate_projection``
    (the bf16 rounding passes gradients unchanged): returns ``dlat`` [B, T, R]
    and, per family, ``dU`` [r, H*d] and ``dbias`` [H*d]."""
    lat = _f64(lat)
    B, T, R = lat.shape
    pre = gate_pre(lat, ups, H)
    dlat = np.zeros_like(lat)
    res = {"dlat": dlat}
    for fam, (off, U, bias) in ups.items():
        U = _f64(U)
        r = U.shape[0]
        dp = (_f64(dgates[GATE_OUTPUT[fam]]) * _gate_act_grad(fam, pre[fam])).reshape(B, T, -1)
        dlat[:, :, off:off + r] += dp @ U.T
        res["dU_" + fam] = np.einsum("bti,btn->in", lat[:, :, off:off + r], dp)
        res["dbias_" + fam] = dp.sum(axis=(0, 1))
    return res
