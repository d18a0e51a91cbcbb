"""CPU checks of the arithmetic devices the kernels use (no GPU needed).

The attention kernel's exact int32 -> fp32 conversion (add the bits of 1.5*2^23, subtract
1.5*2^23) and the prepare kernel's division-free INT8 codes are replayed here in numpy
float32, step by step, and checked against exact integer conversion and exact rounding.
"""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "quantized_block_sparse_b200", "csrc", "attention.cu")
F32 = np.float32


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
