"""GPU parity of the SageSLA backward (sagesla_backward) against oracle/sla_backward_oracle.py.

The oracle differentiates a dense fp64 restatement of the forward with autograd, with the
block lists held fixed and the quantization read straight through (readings B1-B4); it is
pinned by finite differences and by dK's zero sum over tokens. The GPU path computes in
bf16 operands with fp32 accumulation (Q~, K~, V, dO, P, dS, phi and dn rounded to bf16 before
each tensor-core product; softmax statistics, D and the linear denominators in fp32).

Tolerance, per gradient tensor against the fp64 oracle: cosine >= 0.999 and max |error| <=
3e-2 * max |reference|. Each bf16 operand carries a relative rounding error of at most 2^-9;
a product summed over K terms in fp32 then has a relative error of order 2^-9 in the
typical element and a few times that in the worst, and the chain dS = P (dP - D) subtracts
two such quantities, which can lose a further factor where dP and D nearly cancel. The
bound 3e-2 of the tensor's largest element (about 15 bf16 ulps) covers that chain with
margin, and the cosine bound catches systematic errors (a dropped term, a wrong transpose).
At any size, dK must also sum to zero over tokens (the smoothing removes a per-channel
constant from K) within the fp32 rounding of the mean subtraction.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.sla_backward_oracle as G
from quantized_block_sparse_b200 import sagesla as S
from quantized_block_sparse_b200.inputs import WORKLOADS, make_qkv, make_random_qkv
from tests.gpu_helpers import cos, ensure_lib, f32

pytestmark = pytest.mark.gpu

COS_MIN = 0.999
MAXERR_REL = 3e-2


def _run(q, k, v, do, rho, nu):
    ensure_lib()
    B, H, N, _ = q.shape
    qd, kd, vd, dod = (t.cuda().contiguous() for t in (q, k, v, do))
    eng = S.SageSLA(B, H, N, rho, nu)
    eng(qd, kd, vd)
    dq, dk, dv, ws = S.sagesla_backward(qd, kd, vd, dod, eng.prep, eng.sel)
    torch.cuda.synchronize()
    eng.check()
    S.sagesla_check_status(ws)
    return eng, [t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv)]


def _check(q, k, v, do, rho, nu):
    eng, got = _run(q, k, v, do, rho, nu)
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, rho, nu)
    np.testing.assert_array_equal(eng.sel.crit.cpu().numpy(), sel.crit)
    _, ref = G.forward_backward(f32(q), f32(k), f32(v), f32(do), sel)
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        c = cos(g, r)
        err = np.abs(g - r).max()
        assert c >= COS_MIN, (name, c)
        assert err <= MAXERR_REL * np.abs(r).max(), (name, err, np.abs(r).max())
        out[name] = (c, err / np.abs(r).max())
    colsum = np.abs(got[1].sum(axis=2)).max()
    assert colsum <= 1e-4 * np.abs(got[1]).max() * np.sqrt(q.shape[2]), colsum
    return out


def _do(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(torch.bfloat16)


@pytest.mark.parametrize("N,rho,nu", [
    (64, 1.0, 0.0),       # one block, softmax branch only
    (100, 0.5, 0.5),      # ragged, no marginal blocks
    (200, 0.25, 0.25),    # ragged tail with the linear branch on
    (640, 0.3, 0.3),
    (1000, 0.1, 0.45),    # 480p-like ratios at a small size
])
def test_backward_edge_shapes(N, rho, nu):
    q, k, v = make_random_qkv(1, 2, N, seed=N, scale=0.7)
    do = _do(q.shape, N + 1)
    _check(q, k, v, do, rho, nu)


def test_backward_smooth_field_workload():
    wl = WORKLOADS["tiny"]
    q, k, v = make_qkv(wl.B, wl.H, wl.grid, seed=0)
    _check(q, k, v, _do(q.shape, 3), wl.rho, wl.nu)


def test_backward_480p_ratios_mid_size():
    # 480p-like counts and the smooth-field generator at N = 4096 (64 blocks, k_c = 7, m = 28)
    q, k, v = make_qkv(1, 2, (4, 32, 32), seed=5)
    _check(q, k, v, _do(q.shape, 6), 0.1, 0.45)


def test_backward_full_size_480p_properties():
    # The whole 480p layer: finite gradients, dK summing to zero over tokens per channel,
    # and two runs bit-identical (fixed summation orders, no float atomics).
    wl = WORKLOADS["480p"]
    q, k, v = make_qkv(wl.B, wl.H, wl.grid, seed=0)
    do = _do(q.shape, 9)
    ensure_lib()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    eng = S.SageSLA(wl.B, wl.H, wl.N, wl.rho, wl.nu)
    eng(qd, kd, vd)
    a = S.sagesla_backward(qd, kd, vd, dod, eng.prep, eng.sel)
    b = S.sagesla_backward(qd, kd, vd, dod, eng.prep, eng.sel, workspace=a[3])
    torch.cuda.synchronize()
    S.sagesla_check_status(a[3])
    for x, y in zip(a[:3], b[:3]):
        assert torch.isfinite(x).all()
        assert torch.equal(x, y)
    dk = a[1].double()
    colsum = dk.sum(dim=2).abs().max().item()
    assert colsum <= 1e-4 * dk.abs().max().item() * np.sqrt(wl.N), colsum
