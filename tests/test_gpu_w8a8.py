"""GPU parity of the W8A8 block-wise INT8 linear layer against oracle/w8a8_oracle.py.

Bit-exact: the INT8 codes and the fp32 scale bits of both operands (activations and
weights go through the same quantize call).

Tolerance on Y, derived from the kernel's arithmetic (reading W3): each 128-wide K tile's
integer dot product is exact; it is scaled by fl32(s_x * s_w) (relative error <= 2^-24) and
added into an fp32 accumulator by one fused multiply-add (one rounding of <= 2^-24 of the
running sum); the bias is one more fp32 add. With T = sum_kb |s_x s_w dot_kb| + |bias|, the
fp32 result is within (nKT + 2) * 2^-24 * T of the exact value, and rounding it to bf16
adds at most half an ulp, 2^-8 |y|. The test requires every element to meet that bound
against the oracle's fp64 value, and cosine >= 0.99999 overall.
"""
import numpy as np
import pytest
import torch

import oracle.w8a8_oracle as W
from quantized_block_sparse_b200 import sagesla as S
from tests.gpu_helpers import ensure_lib

pytestmark = pytest.mark.gpu


def _abs_terms(x8, sx, w8, sw, bias):
    """T = sum_kb |s_x s_w dot_kb| + |bias| in fp64 (integer dots are exact in fp64 here)."""
    M, K = x8.shape
    N = w8.shape[0]
    rows, cols = np.arange(M) // 128, np.arange(N) // 128
    T = np.zeros((M, N))
    for kb in range(-(-K // 128)):
        ks = slice(kb * 128, min(K, kb * 128 + 128))
        dot = x8[:, ks].astype(np.float64) @ w8[:, ks].astype(np.float64).T
        T += np.abs(dot) * np.abs(sx[rows, kb].astype(np.float64)[:, None] *
                                  sw[cols, kb].astype(np.float64)[None, :])
    if bias is not None:
        T += np.abs(bias.astype(np.float64))[None, :]
    return T


def _check_against_oracle(x, w, bias, rows=None):
    """Quantize x and w on the GPU, run the GEMM, compare (optionally on whole 128-row tiles
    `rows` of x only)."""
    ensure_lib()
    xd, wd = x.cuda(), w.cuda()
    x8, sx = S.sagesla_w8a8_quantize(xd)
    w8, sw = S.sagesla_w8a8_quantize(wd)
    bd = None if bias is None else torch.from_numpy(bias).cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    y = S.sagesla_w8a8_linear(x8, sx, w8, sw, bd, workspace=ws)
    torch.cuda.synchronize()
    S.sagesla_check_status(ws)
    xf, wf = x.float().numpy(), w.float().numpy()
    qx, qsx = W.quantize_tiles(xf)
    qw, qsw = W.quantize_tiles(wf)
    np.testing.assert_array_equal(x8.cpu().numpy(), qx)
    np.testing.assert_array_equal(sx.cpu().numpy().view(np.uint32), qsx.view(np.uint32))
    np.testing.assert_array_equal(w8.cpu().numpy(), qw)
    np.testing.assert_array_equal(sw.cpu().numpy().view(np.uint32), qsw.view(np.uint32))
    g = y.float().cpu().numpy().astype(np.float64)
    if rows is not None:  # whole 128-row tiles: the sub-matrix has the same tiles and scales
        xf, g, qx = xf[rows], g[rows], qx[rows]
        qsx = qsx[np.unique(rows // 128)]
    ref = W.linear(xf, wf, bias)
    nKT = -(-x.shape[1] // 128)
    T = _abs_terms(qx, qsx, qw, qsw, bias)
    bound = (nKT + 2) * 2.0 ** -24 * T * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(ref) + 1e-30
    viol = np.abs(g - ref) > bound
    assert not viol.any(), f"{viol.sum()} elements outside the derived bound"
    c = float((g * ref).sum() / np.sqrt((g * g).sum() * (ref * ref).sum()))
    assert c >= 0.99999, c
    return g, ref


def _operands(M, N, K, seed, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    x[: min(M, 128), : min(K, 128)] *= 8  # tiles with different scales
    bias = (torch.randn(N, generator=g) * 0.1).float().numpy() if with_bias else None
    return x, w, bias


@pytest.mark.parametrize("M,N,K,seed", [
    (128, 128, 128, 0),     # one tile
    (1, 8, 16, 1),          # smallest accepted shape: one row, ragged everything
    (200, 136, 272, 2),     # ragged M, N and K tiles
    (1000, 384, 1536, 3),
    (257, 1544, 1040, 4),   # one-row last M tile, ragged N and K
])
def test_w8a8_ragged_shapes(M, N, K, seed):
    x, w, bias = _operands(M, N, K, seed)
    _check_against_oracle(x, w, bias)


def test_w8a8_no_bias_and_zero_tile():
    x, w, _ = _operands(300, 256, 512, 5, with_bias=False)
    x[128:256, 128:256] = 0  # an all-zero activation tile: s = 0, codes 0
    _check_against_oracle(x, w, None)


@pytest.mark.parametrize("N,K", [(4608, 1536), (1536, 1536), (8960, 1536), (1536, 8960)])
def test_w8a8_wan_1p3b_shapes_sampled(N, K):
    # Wan-1.3B layer shapes at 480p (32760 tokens, hidden 1536): fused QKV, output
    # projection, FFN up and down. Codes and scales are compared whole; Y on three whole
    # 128-row tiles (the first, one inside, and the ragged last of 120 rows).
    M = 32760
    x, w, bias = _operands(M, N, K, 6)
    rows = np.concatenate([np.arange(0, 128), np.arange(128 * 97, 128 * 98), np.arange(128 * 255, M)])
    _check_against_oracle(x, w, bias, rows=rows)


def test_w8a8_two_calls_deterministic():
    x, w, bias = _operands(700, 512, 1024, 7)
    ensure_lib()
    xd, wd = x.cuda(), w.cuda()
    x8, sx = S.sagesla_w8a8_quantize(xd)
    w8, sw = S.sagesla_w8a8_quantize(wd)
    bd = torch.from_numpy(bias).cuda()
    y1 = S.sagesla_w8a8_linear(x8, sx, w8, sw, bd)
    y2 = S.sagesla_w8a8_linear(x8, sx, w8, sw, bd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
