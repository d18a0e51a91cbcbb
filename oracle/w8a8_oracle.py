"""CPU oracle for the W8A8 block-wise INT8 linear layer.  TEST INFRASTRUCTURE ONLY.

Only the tests may import this module. It shares no code, table or helper with any CUDA
kernel.

What it computes:

* "TurboDiffusion Demystified: How It Achieves 100x Faster Video Generation", section
  "Pillar Three: W8A8 Linear Layer Quantization": the linear (fully connected) layers
  quantize both weights and activations to INT8, at a block-wise granularity of 128x128.
* "TurboDiffusion: Genombrottet för realtids AI-videogenerering", section "W8A8
  Quantization": the whole model runs with 8-bit weights and activations.

The pages fix nothing beyond that. The readings taken here, in their plainest form:

1. Granularity. Both operands are cut into 128x128 tiles: the activations X [M, K] by
   (128 rows, 128 input channels) and the weights W [N, K] by (128 output channels, 128
   input channels). Edge tiles are ragged.
2. Per tile, symmetric INT8 with a stored fp32 scale, exactly as for attention:
   s = fl32(max|x| / 127), x8 = clamp(rint(fl32(x / s)), -127, 127), with rint rounding
   half to even. An all-zero tile gives s = 0 and x8 = 0.
3. Y = X W^T + bias, computed as a sum over the 128-wide input-channel tiles kb:
   Y[m, n] = sum_kb s_x[m/128, kb] * s_w[n/128, kb] * sum_{k in kb} x8[m, k] * w8[n, k].
   Each inner sum is an exact integer. Here the scaling and the sum over kb are fp64.
   The bias, when present, is added last. The output is rounded once to bf16.

Pinned by CPU tests against exactly representable inputs (the codes and scales are then
known in closed form, and Y equals the plain product), against brute-force loops on
ragged shapes, and against the quantization error bound.
"""
from __future__ import annotations

import numpy as np

from .sagesla_oracle import round_bf16

TILE = 128
_F32 = np.float32


def _tiles(n: int) -> int:
    return -(-n // TILE)


def quantize_tiles(x: np.ndarray):
    """Symmetric INT8 per 128x128 tile (reading 2).

    x is a 2-D array, rounded to fp32 first. Returns (x8 int8 of x's shape, s fp32 of
    shape [ceil(R/128), ceil(C/128)]).
    """
    x = np.asarray(x, dtype=_F32)
    R, C = x.shape
    tr, tc = _tiles(R), _tiles(C)
    xp = np.zeros((tr * TILE, tc * TILE), dtype=_F32)
    xp[:R, :C] = x
    t = xp.reshape(tr, TILE, tc, TILE)
    amax = np.abs(t).max(axis=(1, 3)).astype(_F32)  # padding is 0, so it never wins
    s = (amax / _F32(127.0)).astype(_F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (t / s[:, None, :, None]).astype(_F32)
    y = np.where(s[:, None, :, None] > 0, y, _F32(0))
    x8 = np.clip(np.rint(y), -127, 127).astype(np.int8)
    return x8.reshape(tr * TILE, tc * TILE)[:R, :C], s


def dequantize_tiles(x8: np.ndarray, s: np.ndarray) -> np.ndarray:
    """x8 * s per tile, in fp64 (exact: an 8-bit code times an fp32 scale)."""
    R, C = x8.shape
    rows = np.arange(R) // TILE
    cols = np.arange(C) // TILE
    return x8.astype(np.float64) * s.astype(np.float64)[rows[:, None], cols[None, :]]


def linear(x: np.ndarray, w: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """Y = X W^T (+ bias) with both operands quantized per 128x128 tile (reading 3).

    x: [M, K], w: [N, K], bias: [N] or None. Returns fp64 [M, N] before the bf16 rounding.
    """
    x8, sx = quantize_tiles(x)
    w8, sw = quantize_tiles(w)
    M, K = x8.shape
    N, K2 = w8.shape
    if K != K2:
        raise ValueError("x and w disagree on the input width")
    mrow = np.arange(M) // TILE
    ncol = np.arange(N) // TILE
    y = np.zeros((M, N), dtype=np.float64)
    for kb in range(_tiles(K)):
        ks = slice(kb * TILE, min(K, (kb + 1) * TILE))
        acc = x8[:, ks].astype(np.int64) @ w8[:, ks].astype(np.int64).T  # exact
        scale = (sx[mrow, kb].astype(np.float64)[:, None] *
                 sw[ncol, kb].astype(np.float64)[None, :])
        y += acc.astype(np.float64) * scale
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)[None, :]
    return y


def w8a8_linear(x, w, bias=None) -> np.ndarray:
    """The layer's output: linear() rounded once to bf16 (fp64 array of bf16 values)."""
    return round_bf16(linear(x, w, bias))
