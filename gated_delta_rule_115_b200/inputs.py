"""Seeded synthetic inputs for the Muir gated delta rule.

This module only draws random numbers and shapes them into the input
distributions of the workloads; it contains none of the recurrence's
arithmetic.  Tests, ``bench.py`` and the oracle side of the tests all take
their inputs from here, so both sides see the same values.

Recipe (stated once, used everywhere):

* ``torch.Generator('cpu').manual_seed(seed)``, default ``seed = 1000 + workload
  id``; draws in float32 in the fixed order q, k, v, g, e, w, gamma, S0, dO;
  then one round-to-nearest-even cast to the workload dtype (bf16 or fp32).
  States (S0) stay float32.
* q, k = L2-normalise(SiLU(N(0,1))) over the key channels.
* v ~ N(0,1).
* g = -softplus(N(0,1)) per key channel and token (log decay, always <= 0).
* e, w, gamma = sigmoid(N(0,1)) per channel and token, except:
  - ``gates="proj"``: e and w come from a seeded low-rank projection of a
    random d_model = 2048 input: x ~ N(0,1) [B,T,2048], a shared down-projection
    W_down ~ N(0, 1/2048) [2048, 64+128], up-projections W_e ~ N(0,1/64)
    [64, H*dk] and W_w ~ N(0,1/128) [128, H*dv], channel biases ~ N(0,1) per
    (h, channel); e = sigmoid(x W_down[:, :64] W_e + b_e),
    w = sigmoid(x W_down[:, 64:] W_w + b_w).  Ranks 64 (erase) and 128 (write)
    follow the gate ranks listed for Muir (wolonglab.org page, fig:arch,
    "Methodology"); no nonlinearity inside the bottleneck.
  - ``gates="stress"``: g is drawn once per (b, h, channel), uniform in
    [-8, -1e-4], and held constant over tokens (slow and fast rows mixed);
    e = 1 on a Bernoulli(0.1) subset of (b, h, channel), constant over tokens,
    else sigmoid(N(0,1)) per token.
* S0 = 0, or N(0, s^2) with the workload's s (sqrt(10) for the stress case).
* dO ~ N(0,1).

Decode: the state S0 ~ N(0,1) float32 and a static gamma [H, dk] come from the
base generator; the tokens of step ``i`` come from their own generator seeded
with ``seed * 1_000_003 + i + 1``, so any step can be regenerated alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str  # "bf16" | "fp32"
    gates: str = "iid"  # "iid" | "proj" | "stress"
    s0_std: float = 0.0
    with_dO: bool = False
    steps: int = 0  # decode steps (decode workload only)
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    0: Workload(0, "tiny fp32 forward (B=1,H=2,T=256,d=64,C=64)", 1, 2, 256, 64, 64, 64,
                "fp32", with_dO=True),
    1: Workload(1, "layer-shaped bf16 forward (B=8,H=16,T=4096,d=128,C=64)", 8, 16, 4096,
                128, 128, 64, "bf16", gates="proj"),
    2: Workload(2, "long-context bf16 fwd+bwd (B=1,H=16,T=32768,d=128,C=128)", 1, 16, 32768,
                128, 128, 128, "bf16", gates="proj", with_dO=True),
    3: Workload(3, "large-chunk stress bf16 (B=2,H=8,T=8192,d=128,C=256)", 2, 8, 8192, 128,
                128, 256, "bf16", gates="stress", s0_std=math.sqrt(10.0)),
    4: Workload(4, "streaming decode (B=64,H=16,d=128, fp32 state)", 64, 16, 1, 128, 128, 1,
                "bf16", steps=10000),
}

TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}


def _randn(gen, *shape):
    return torch.randn(*shape, generator=gen, dtype=torch.float32)


def _unit_keys(x):
    x = F.silu(x)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def chunk_inputs(wid: int, *, B=None, H=None, T=None, dk=None, dv=None, seed=None,
                 dtype=None, gates=None, s0_std=None, with_dO=None):
    """Inputs of a chunked workload as CPU tensors.

    Returns a dict with q, k, v, g, e, w, gamma (``[B,T,H,d]``, workload dtype),
    S0 (``[B,H,dk,dv]`` float32, or None for a zero state) and dO (or None).
    Any shape or recipe field can be overridden for small test cases.
    """
    W = WORKLOADS[wid]
    B = W.B if B is None else B
    H = W.H if H is None else H
    T = W.T if T is None else T
    dk = W.dk if dk is None else dk
    dv = W.dv if dv is None else dv
    dtype = W.dtype if dtype is None else dtype
    gates = W.gates if gates is None else gates
    s0_std = W.s0_std if s0_std is None else s0_std
    with_dO = W.with_dO if with_dO is None else with_dO
    seed = 1000 + wid if seed is None else seed
    gen = torch.Generator("cpu").manual_seed(seed)

    q = _unit_keys(_randn(gen, B, T, H, dk))
    k = _unit_keys(_randn(gen, B, T, H, dk))
    v = _randn(gen, B, T, H, dv)
    if gates == "stress":
        g = (torch.rand(B, 1, H, dk, generator=gen) * (-1e-4 + 8.0) - 8.0).expand(B, T, H, dk)
    else:
        g = -F.softplus(_randn(gen, B, T, H, dk))
    if gates == "proj":
        x = _randn(gen, B, T, 2048)
        w_down = _randn(gen, 2048, 64 + 128) / math.sqrt(2048.0)
        w_e = _randn(gen, 64, H * dk) / math.sqrt(64.0)
        b_e = _randn(gen, H * dk)
        z = x.reshape(B * T, 2048) @ w_down
        e = torch.sigmoid(z[:, :64] @ w_e + b_e).reshape(B, T, H, dk)
        w_w = _randn(gen, 128, H * dv) / math.sqrt(128.0)
        b_w = _randn(gen, H * dv)
        w = torch.sigmoid(z[:, 64:] @ w_w + b_w).reshape(B, T, H, dv)
        del x, z
    elif gates == "stress":
        mask = torch.rand(B, 1, H, dk, generator=gen) < 0.1
        e = torch.where(mask, torch.ones(()), torch.sigmoid(_randn(gen, B, T, H, dk)))
        w = torch.sigmoid(_randn(gen, B, T, H, dv))
    else:
        e = torch.sigmoid(_randn(gen, B, T, H, dk))
        w = torch.sigmoid(_randn(gen, B, T, H, dv))
    gamma = torch.sigmoid(_randn(gen, B, T, H, dk))
    S0 = _randn(gen, B, H, dk, dv) * s0_std if s0_std > 0 else None
    dO = _randn(gen, B, T, H, dv) if with_dO else None

    td = TORCH_DTYPE[dtype]
    out = {n: t.contiguous().to(td) for n, t in
           dict(q=q, k=k, v=v, g=g, e=e, w=w, gamma=gamma).items()}
    out["S0"] = S0.contiguous() if S0 is not None else None
    out["dO"] = dO.to(td).contiguous() if dO is not None else None
    return out


def decode_state(wid: int = 4, *, B=None, H=None, dk=None, dv=None, seed=None):
    """Initial state S0 ~ N(0,1) [B,H,dk,dv] float32 and static gamma [H,dk]
    (= sigmoid(N(0,1)), in the workload dtype) of the decode workload."""
    W = WORKLOADS[wid]
    B = W.B if B is None else B
    H = W.H if H is None else H
    dk = W.dk if dk is None else dk
    dv = W.dv if dv is None else dv
    seed = 1000 + wid if seed is None else seed
    gen = torch.Generator("cpu").manual_seed(seed)
    gamma = torch.sigmoid(_randn(gen, H, dk)).to(TORCH_DTYPE[W.dtype])
    S0 = _randn(gen, B, H, dk, dv)
    return S0.contiguous(), gamma.contiguous()


def decode_tokens(step: int, wid: int = 4, *, B=None, H=None, dk=None, dv=None, seed=None,
                  dtype=None):
    """Tokens of decode step ``step``: q, k, v, g, e, w as ``[B,H,d]`` tensors."""
    W = WORKLOADS[wid]
    B = W.B if B is None else B
    H = W.H if H is None else H
    dk = W.dk if dk is None else dk
    dv = W.dv if dv is None else dv
    dtype = W.dtype if dtype is None else dtype
    seed = 1000 + wid if seed is None else seed
    gen = torch.Generator("cpu").manual_seed(seed * 1_000_003 + step + 1)
    q = _unit_keys(_randn(gen, B, H, dk))
    k = _unit_keys(_randn(gen, B, H, dk))
    v = _randn(gen, B, H, dv)
    g = -F.softplus(_randn(gen, B, H, dk))
    e = torch.sigmoid(_randn(gen, B, H, dk))
    w = torch.sigmoid(_randn(gen, B, H, dv))
    td = TORCH_DTYPE[dtype]
    return {n: t.to(td).contiguous() for n, t in
            dict(q=q, k=k, v=v, g=g, e=e, w=w).items()}


def fused_inputs(wid: int, *, seed=None, **over):
    """Inputs of the fused layer: those of :func:`chunk_inputs` (same
    overrides), plus raw q/k pre-activations ``xq``, ``xk`` ~ N(0,1) (the
    prologue's inputs) and the output gate's pre-activation ``z_out`` ~ N(0,1),
    all ``[B,T,H,d]`` in the workload dtype, drawn from their own seed."""
    x = chunk_inputs(wid, **over)
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    gen = torch.Generator("cpu").manual_seed((5000 + wid) if seed is None else seed)
    td = x["q"].dtype
    x["xq"] = _randn(gen, B, T, H, dk).to(td).contiguous()
    x["xk"] = _randn(gen, B, T, H, dk).to(td).contiguous()
    x["z_out"] = _randn(gen, B, T, H, dv).to(td).contiguous()
    return x


GATE_RANKS = {"f": 64, "b": 64, "g": 128, "w": 128, "q": 128}  # (r_f, r_b, r_g, r_w, r_q)


def gate_latent_inputs(B: int, T: int, H: int, d: int = 128, *, seed=None, dtype="bf16",
                       families=("f", "b", "g", "w", "q"), bias_f=-2.5):
    """Parameters of the fused gate projection: a per-token latent
    ``[B, T, R]`` ~ N(0,1) (R = 512, families laid out in the order f, b, g, w,
    q with ranks 64, 64, 128, 128, 128), per family an up-projection
    ``U [r, H*d]`` ~ N(0, 1/r) (so pre-activations are ~N(0,1)) and a channel
    bias ~ N(0, 0.25) in float32 (the decay family's centred at ``bias_f``: at
    -2.5 every chunk's per-channel log-decay total at B=1, H=16, T=32768 stays
    within 105, inside the single-pivot range like the long-context workload's
    134; the bias persists over tokens, so per-channel totals spread wider than
    with iid gates).  Returns ``(latent, {family: (offset, U,
    bias)})`` as CPU tensors."""
    gen = torch.Generator("cpu").manual_seed(7000 if seed is None else seed)
    td = TORCH_DTYPE[dtype]
    R = sum(GATE_RANKS.values())
    lat = _randn(gen, B, T, R).to(td).contiguous()
    proj, off = {}, 0
    for fam in ("f", "b", "g", "w", "q"):
        r = GATE_RANKS[fam]
        U = (_randn(gen, r, H * d) / math.sqrt(r)).to(td).contiguous()
        bias = _randn(gen, H * d) * 0.5 + (bias_f if fam == "f" else 0.0)
        if fam in families:
            proj[fam] = (off, U, bias.contiguous())
        off += r
    return lat, proj
