"""Parity of the CUDA q/k prologue (muir_qk_prologue / muir_qk_prologue_bwd)
against the fp64 oracle on seeded inputs.

Error metric: max |gpu - oracle| / max |oracle| per tensor.  Both sides read
the same stored inputs.  Tolerances from the arithmetic: the kernel's sigmoid
uses the fast exponential (at most 2 + 1.173|x| ulp) and division (2 ulp), so
for the |x| <= 10 that carry a row's weight sigmoid is within 15 ulp (~9e-7
relative), SiLU and the normalised row within about 2e-6: float32 outputs 5e-6
(forward) and 1e-5 (backward, one more sigmoid and the cancellation
dy - y (y . dy)); bfloat16 outputs are rounded once to nearest even, a
relative error of at most 2^-8 per element, so 4e-3 (forward) and 5e-3
(backward).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL_FWD = {torch.float32: 5e-6, torch.bfloat16: 4e-3}
TOL_BWD = {torch.float32: 1e-5, torch.bfloat16: 5e-3}


@pytest.fixture(scope="module")
def muir():
    import gated_delta_rule_115_b200 as m
    m.lib()
    return m


def nmax(a, r):
    a = a.double().cpu().numpy()
    return float(np.abs(a - r).max() / max(np.abs(r).max(), 1e-300))


def rows_input(rows, d, dtype, seed):
    """N(0,1) rows, with a zero row, a row of large negative values (SiLU
    underflows: the norm guard takes over), and rows of large magnitude."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, d, generator=g)
    if rows > 3:
        x[1] = 0.0
        x[2] = -90.0
        x[3] = 30.0 * torch.randn(d, generator=g)
    return x.to(dtype)


CASES = [(r, d, dt) for d in (64, 128) for dt in (torch.bfloat16, torch.float32)
         for r in (1, 37, 4099)]


@pytest.mark.parametrize("rows,d,dtype", CASES)
def test_qk_prologue_parity(muir, oracle_mod, rows, d, dtype):
    x = rows_input(rows, d, dtype, 10 + rows + d)
    y = muir.qk_prologue(x.cuda())
    r = oracle_mod.qk_prologue(x)
    torch.cuda.synchronize()
    e = nmax(y, r)
    print(f"qk fwd rows={rows} d={d} {dtype}: {e:.2e}")
    assert y.dtype == dtype and e < TOL_FWD[dtype]


@pytest.mark.parametrize("rows,d,dtype", CASES)
def test_qk_prologue_bwd_parity(muir, oracle_mod, rows, d, dtype):
    x = rows_input(rows, d, dtype, 20 + rows + d)
    dy = torch.randn(rows, d, generator=torch.Generator().manual_seed(rows)).to(dtype)
    if rows > 3:
        dy[1] = 0.0  # the zero row's gradient is dy / (2 eps): keep it finite and comparable
    dx = muir.qk_prologue_bwd(x.cuda(), dy.cuda())
    r = oracle_mod.qk_prologue_bwd(x, dy)
    torch.cuda.synchronize()
    e = nmax(dx, r)
    print(f"qk bwd rows={rows} d={d} {dtype}: {e:.2e}")
    assert e < TOL_BWD[dtype]


def test_qk_prologue_in_place_and_empty(muir):
    x = rows_input(300, 128, torch.bfloat16, 5).cuda()
    y = muir.qk_prologue(x)
    z = x.clone()
    muir.qk_prologue(z, out=z)
    assert torch.equal(y, z)
    e = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    assert muir.qk_prologue(e).numel() == 0


def test_qk_prologue_full_size(muir, oracle_mod):
    """The long-context workload's q (B=1, T=32768, H=16, d=128, bf16) in one
    call: every row has unit norm (up to bf16 storage), sampled rows match the
    oracle, and the backward of sampled rows matches too."""
    g = torch.Generator().manual_seed(7)
    x = torch.randn(1, 32768, 16, 128, generator=g).to(torch.bfloat16)
    xd = x.cuda()
    y = muir.qk_prologue(xd)
    dy = torch.randn(1, 32768, 16, 128, generator=g).to(torch.bfloat16)
    dx = muir.qk_prologue_bwd(xd, dy.cuda())
    torch.cuda.synchronize()
    nrm = y.float().norm(dim=-1)
    assert (nrm - 1.0).abs().max().item() < 1e-2
    rows = np.random.default_rng(0).choice(32768 * 16, 512, replace=False)
    xr = x.reshape(-1, 128)[rows]
    assert nmax(y.reshape(-1, 128)[rows], oracle_mod.qk_prologue(xr)) < TOL_FWD[torch.bfloat16]
    rb = oracle_mod.qk_prologue_bwd(xr, dy.reshape(-1, 128)[rows])
    assert nmax(dx.reshape(-1, 128)[rows], rb) < TOL_BWD[torch.bfloat16]
