"""Pins for the W8A8 block-wise INT8 linear oracle (oracle/w8a8_oracle.py), CPU only.

Each pin checks the oracle against something other than its own formulas: inputs whose
codes and scales are known in closed form, a different evaluation order (dequantize, then
one fp64 product), and the quantization error bound against the plain product. The last
tests plant plausible mistakes in the oracle and check that a pin catches each.
"""
import numpy as np
import pytest

import oracle.w8a8_oracle as W

T = W.TILE


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def _coded(rng, R, C, exps):
    """x = q * 2^e per 128x128 tile, every tile holding a +-127 code: the scale is 2^e and
    the codes are q exactly. exps[i][j] is the tile's exponent (None: an all-zero tile)."""
    q = rng.integers(-127, 128, size=(R, C))
    s = np.zeros((-(-R // T), -(-C // T)))
    x = np.zeros((R, C))
    for i in range(s.shape[0]):
        for j in range(s.shape[1]):
            rs, cs = slice(i * T, min(R, (i + 1) * T)), slice(j * T, min(C, (j + 1) * T))
            if exps[i][j] is None:
                q[rs, cs] = 0
                continue
            q[rs.start, cs.start] = 127 if (i + j) % 2 == 0 else -127
            s[i, j] = 2.0 ** exps[i][j]
            x[rs, cs] = q[rs, cs] * s[i, j]
    return x.astype(np.float32), q.astype(np.int8), s.astype(np.float32)


def test_codes_and_scales_closed_form():
    rng = np.random.default_rng(0)
    exps = [[-3, 0, None], [2, -7, 1]]
    x, q, s = _coded(rng, 200, 300, exps)  # ragged in both dimensions
    x8, sx = W.quantize_tiles(x)
    assert sx.shape == (2, 3) and sx.dtype == np.float32
    np.testing.assert_array_equal(sx, s)
    np.testing.assert_array_equal(x8, q)


def test_codes_round_half_to_even():
    s = 2.0 ** -4
    x = np.zeros((T, T), dtype=np.float32)
    x[0, 0] = 127 * s                      # fixes the scale at s
    halves = np.arange(12) + 0.5           # 0.5, 1.5, ..., 11.5 (exact multiples of s/2)
    x[1, :12] = halves * s
    x[2, :12] = -halves * s
    x8, sx = W.quantize_tiles(x)
    assert sx[0, 0] == np.float32(s)
    even = np.array([0, 2, 2, 4, 4, 6, 6, 8, 8, 10, 10, 12])
    np.testing.assert_array_equal(x8[1, :12], even)
    np.testing.assert_array_equal(x8[2, :12], -even)


def test_linear_exact_on_representable_inputs():
    rng = np.random.default_rng(1)
    x, _, _ = _coded(rng, 130, 257, [[-2, 1, 0], [3, None, -1]])
    w, _, _ = _coded(rng, 140, 257, [[0, -3, 2], [1, 2, -2]])
    bias = (rng.integers(-64, 64, size=140) * 0.25).astype(np.float32)
    y = W.linear(x, w, bias)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + bias.astype(np.float64)[None, :]
    np.testing.assert_array_equal(y, ref)


def test_linear_equals_dequantized_product():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((193, 300)).astype(np.float32) * 3
    w = rng.standard_normal((70, 300)).astype(np.float32)
    x[:, 200:] *= 50  # tiles with different scales along the input width
    y = W.linear(x, w)
    xd = W.dequantize_tiles(*W.quantize_tiles(x))
    wd = W.dequantize_tiles(*W.quantize_tiles(w))
    np.testing.assert_allclose(y, xd @ wd.T, rtol=1e-12, atol=1e-9)


def test_linear_within_quantization_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((256, 384)).astype(np.float32)
    w = rng.standard_normal((130, 384)).astype(np.float32)
    x[:128, :128] *= 20.0
    w[128:, 256:] *= 0.01
    y = W.linear(x, w)
    ex = _code_error(x)
    ew = _code_error(w)
    ax, aw = np.abs(x.astype(np.float64)), np.abs(w.astype(np.float64))
    bound = ax @ ew.T + ex @ aw.T + ex @ ew.T
    err = np.abs(y - x.astype(np.float64) @ w.astype(np.float64).T)
    assert (err <= bound * (1 + 1e-9) + 1e-12).all()
    assert err.max() > 0  # the bound is not met trivially


def _code_error(x):
    """Per-element bound on |x - s*x8|: half a step plus the fp32 rounding of x/s."""
    _, s = W.quantize_tiles(x)
    R, C = x.shape
    st = s.astype(np.float64)[(np.arange(R) // T)[:, None], (np.arange(C) // T)[None, :]]
    return st * (0.5 + 127 * 2.0 ** -24)


def test_zero_tile_and_shapes():
    x = np.zeros((5, 7), dtype=np.float32)
    x8, s = W.quantize_tiles(x)
    assert (x8 == 0).all() and (s == 0).all()
    w = np.ones((3, 7), dtype=np.float32)
    np.testing.assert_array_equal(W.linear(x, w, np.arange(3, dtype=np.float32)),
                                  np.broadcast_to(np.arange(3.0), (5, 3)))
    with pytest.raises(ValueError):
        W.linear(np.ones((2, 8), np.float32), np.ones((2, 7), np.float32))


def test_output_rounded_once_to_bf16():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    w = rng.standard_normal((32, 128)).astype(np.float32)
    y = W.w8a8_linear(x, w)
    y32 = W.linear(x, w).astype(np.float32)
    bits = y.astype(np.float32).view(np.uint32)
    assert (bits & 0xFFFF == 0).all()  # bf16 values
    ulp = np.abs(y32.view(np.uint32).astype(np.int64) - bits.astype(np.int64))
    assert (ulp <= 0x8000).all()        # within half a bf16 step of the fp32 value


# ---- planted mistakes: each must make one of the pins above fail

def test_mutation_per_row_scale(monkeypatch):
    orig = W.quantize_tiles

    def per_row(x):
        x = np.asarray(x, dtype=np.float32)
        x8, s = orig(x)
        amax = np.abs(x).max(axis=1, keepdims=True)
        sr = (amax / np.float32(127)).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(sr > 0, np.rint(x / sr), 0)
        return np.clip(q, -127, 127).astype(np.int8), s

    monkeypatch.setattr(W, "quantize_tiles", per_row)
    assert _fails(test_codes_and_scales_closed_form)


def test_mutation_truncated_codes(monkeypatch):
    orig = W.quantize_tiles

    def truncating(x):
        x = np.asarray(x, dtype=np.float32)
        x8, s = orig(x)
        R, C = x.shape
        st = s[(np.arange(R) // T)[:, None], (np.arange(C) // T)[None, :]]
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(st > 0, np.trunc(x / st), 0)
        return q.astype(np.int8), s

    monkeypatch.setattr(W, "quantize_tiles", truncating)
    assert _fails(test_codes_round_half_to_even)


def test_mutation_weight_scale_ignores_k_tile(monkeypatch):
    # the weight scale of the first input-channel tile applied to every tile
    def one_scale_per_row_block(x, w, bias=None):
        x8, sx = W.quantize_tiles(x)
        w8, sw = W.quantize_tiles(w)
        M, K = x8.shape
        N = w8.shape[0]
        mrow, ncol = np.arange(M) // T, np.arange(N) // T
        y = np.zeros((M, N))
        for kb in range(-(-K // T)):
            ks = slice(kb * T, min(K, (kb + 1) * T))
            acc = x8[:, ks].astype(np.int64) @ w8[:, ks].astype(np.int64).T
            y += acc * (sx[mrow, kb].astype(np.float64)[:, None] * sw[ncol, 0].astype(np.float64)[None, :])
        return y + (0 if bias is None else np.asarray(bias, np.float64)[None, :])

    monkeypatch.setattr(W, "linear", one_scale_per_row_block)
    assert _fails(test_linear_exact_on_representable_inputs)


def test_mutation_bias_dropped(monkeypatch):
    orig = W.linear
    monkeypatch.setattr(W, "linear", lambda x, w, bias=None: orig(x, w, None))
    assert _fails(test_linear_exact_on_representable_inputs)
