"""GPU parity of the marginal gather-sum on its own (the first half of step 6, "TurboDiffusion
Demystified", section "Pillar Two: Sparse-Linear Attention - SLA"): H_i = sum of h_j and
Z_i = sum of z_j over the marginal key blocks j of query block i.

The reference is that definition in fp64 on the kernel's own inputs (h, z from prepare, the
mask from select), so the mask GEMM is checked alone: each product of a 0/1 mask entry and a
bf16 value is exact, the tensor core sums them in fp32 and H is rounded once to bf16, so H
is within one bf16 ulp of the exact sum plus the fp32 summation bound; Z is the fp32 sum of
z's two bf16 parts, within 2^-15 of the exact sum plus the same bound.
"""
import numpy as np
import pytest
import torch

from quantized_block_sparse_b200 import sagesla as S
from quantized_block_sparse_b200.inputs import make_random_qkv
from tests.gpu_helpers import ensure_lib

pytestmark = pytest.mark.gpu


def _bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 0.0)


@pytest.mark.parametrize("N,rho,nu", [
    (1000, 0.25, 0.25),  # ragged tail, m = 8
    (2000, 0.1, 0.45),   # 480p-like ratios at a small size
    (150, 0.25, 0.3),    # three blocks, one marginal per row
    (100, 0.5, 0.5),     # no marginal block (m = 0): H and Z are zero
    (8192, 0.1, 0.45),   # 128 blocks: a full 128-row tile and several k-blocks of the GEMM
])
def test_marginal_sums_match_their_definition(N, rho, nu):
    ensure_lib()
    q, k, v = make_random_qkv(1, 2, N, seed=N + 7)
    eng = S.SageSLA(1, 2, N, rho, nu)
    eng(q.cuda(), k.cuda(), v.cuda())
    sel, prep = eng.sel, eng.prep
    Hg, Zg = S.sagesla_marginal_sums(sel.mask, sel.m, prep.h, prep.z, eng.workspace, N=N)
    torch.cuda.synchronize()
    eng.check()
    nB = prep.h.shape[2]
    M = sel.mask.double().cpu().numpy()[..., :nB]
    h = prep.h.double().cpu().numpy()
    z = prep.z.double().cpu().numpy()
    Hx = np.einsum("bhij,bhjcd->bhicd", M, h)
    Zx = np.einsum("bhij,bhjc->bhic", M, z)
    Hg = Hg.double().cpu().numpy()
    Zg = Zg.double().cpu().numpy()
    # fp32 summation bound over at most m terms (every partial sum below m * max|x|)
    eh = sel.m * 2.0 ** -24 * np.abs(h).max() * max(sel.m, 1)
    ez = sel.m * 2.0 ** -24 * np.abs(z).max() * max(sel.m, 1)
    assert (np.abs(Hg - Hx) <= _bf16_ulp(Hx) + eh).all()
    assert (np.abs(Zg - Zx) <= 2.0 ** -15 * np.abs(Zx) + ez).all()
    if sel.m == 0:
        assert not Hg.any() and not Zg.any()
    else:
        assert (M.sum(axis=-1) == sel.m).all()  # every row sums exactly m blocks
