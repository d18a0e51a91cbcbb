"""CPU checks of the arithmetic devices the attention kernel uses (no GPU needed).

The kernel's FMA-pipe exp2 (range reduction x = rint(x) + f, degree-3 polynomial for 2^f,
exponent-field add) and its exact int32 -> fp32 conversion (add the bits of 1.5*2^23,
subtract 1.5*2^23) are replayed here in numpy float32, step by step, and checked against
exp2 in float64 and against exact integer conversion.
"""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "quantized_block_sparse_b200", "csrc", "attention.cu")
F32 = np.float32


def _coeffs():
    """The four polynomial constants, read from the kernel source."""
    text = open(SRC).read()
    body = text[text.index("void exp2_poly2"):text.index("y0 = __int_as_float")]
    vals = [float(v) for v in re.findall(r"f2pack\(([0-9.]+)f, \1f\)", body)]
    assert len(vals) == 4
    c3, c2, c1, c0 = vals
    return F32(c0), F32(c1), F32(c2), F32(c3)


def _fma32(a, b, c):
    # fp32 fused multiply-add: the product of two float32 is exact in float64; the sum is
    # rounded once to float64 then to float32 (close enough for these bounds).
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def exp2_poly_replay(x):
    c0, c1, c2, c3 = _coeffs()
    M = F32(12582912.0)
    x = np.maximum(x.astype(F32), F32(-125.0))
    t = (x + M).astype(F32)
    n = (t - M).astype(F32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF)
    bits = ((bits + 2 ** 31) % 2 ** 32 - 2 ** 31).astype(np.int32)
    return bits.view(F32)


def test_exp2_poly_relative_error():
    x = np.concatenate([np.linspace(-125, 9, 400001), np.linspace(-1, 1, 100001)]).astype(F32)
    y = exp2_poly_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() < 1e-4, rel.max()  # far below the 2^-9 rounding of bf16 P


def test_exp2_poly_rounding_boundaries_and_clamp():
    # half-integers (tie cases of rint) and integers are continuous / exact-ish
    x = np.array([-3.5, -2.5, -0.5, 0.5, 1.5, 2.5, 0.0, 1.0, 8.0, -126.0, -1000.0], dtype=F32)
    y = exp2_poly_replay(x).astype(np.float64)
    ref = np.exp2(np.maximum(x.astype(np.float64), -125.0))
    assert (np.abs(y / ref - 1) < 1e-4).all()
    assert y[-1] > 0 and y[-1] < 1e-37  # clamped: tiny, never a wrapped exponent


def test_magic_int_to_float_is_exact():
    v = np.concatenate([np.arange(-2 ** 21, 2 ** 21, 997), [-128 * 127 * 127, 128 * 127 * 127, 0, 1, -1]])
    bits = (v.astype(np.int64) + 0x4B400000).astype(np.int32)
    f = (bits.view(F32) - F32(12582912.0)).astype(F32)
    np.testing.assert_array_equal(f.astype(np.int64), v)
    # and the order of the offset floats is the order of the integers (row max on floats)
    assert (np.diff(bits.view(F32)[np.argsort(v)]) >= 0).all()


# ---------------------------------------------------------------------------------------
# Division-free INT8 codes (prepare): rint(fl32(x*fl32(1/s))) with an exact-division
# fallback within a band around half-integers. Replayed in float32 and compared with
# rint(fl32(x/s)), the definition the oracle uses.
PREP = os.path.join(os.path.dirname(SRC), "prepare.cu")


def _prep_threshold():
    text = open(PREP).read()
    body = text[text.index("uint64_t quant_pair("):]
    m = re.search(r"fabsf\(e\.x\) > ([0-9.]+)f \|\| fabsf\(e\.y\) > ([0-9.]+)f", body)
    assert m.group(1) == m.group(2)  # both lanes of the pair use one band
    return F32(float(m.group(1)))


def quant_byte_replay(x, s):
    thr = _prep_threshold()
    M = F32(12582912.0)
    rs = (F32(1.0) / s).astype(F32)
    y = (x * rs).astype(F32)
    t = (y + M).astype(F32)
    e = ((t - M).astype(F32) - y).astype(F32)
    code = (t.view(np.uint32) & 0xFF).astype(np.int64)
    code = np.where(code > 127, code - 256, code)
    exact = np.clip(np.rint((x / s).astype(F32)), -127, 127).astype(np.int64)
    return np.where(np.abs(e) > thr, exact, code), np.abs(e) > thr


def test_division_free_codes_match_exact_rounding():
    rng = np.random.default_rng(5)
    for _ in range(60):
        amax = F32(np.exp(rng.uniform(-30, 12)))
        s = F32(amax / F32(127.0))
        x = (rng.uniform(-1, 1, 50000) * amax).astype(F32)
        # quotients planted next to half-integers, within a few ulps
        h = rng.integers(-127, 127, 50000) + 0.5
        x2 = np.clip((h * np.float64(s) * (1 + rng.uniform(-4e-7, 4e-7, 50000))).astype(F32), -amax, amax)
        xx = np.concatenate([x, x2, np.array([amax, -amax, 0.0], F32)])
        got, fell_back = quant_byte_replay(xx, s)
        want = np.clip(np.rint((xx / s).astype(F32)), -127, 127).astype(np.int64)
        np.testing.assert_array_equal(got, want)
        assert fell_back[:50000].mean() < 1e-3  # ordinary values almost never divide
