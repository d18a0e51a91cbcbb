"""Pins for the CPU oracle: each check ties it to something other than itself.

Closed forms, invariances, library routines (torch SDPA, torch elu, numpy sorts) and
brute force on tiny inputs. No GPU needed.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from quantized_block_sparse_b200.inputs import make_qkv, make_random_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(t):
    return t.float().numpy()


def sdpa64(q, k, v, scale):
    """fp64 full softmax attention by torch's library routine."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.as_tensor(q, dtype=torch.float64), torch.as_tensor(k, dtype=torch.float64),
        torch.as_tensor(v, dtype=torch.float64), scale=float(scale)).numpy()


def cos(a, b):
    a = a.reshape(-1)
    b = b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


# ------------------------------------------------------------------ counts
def test_counts_golden_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "counts.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for nB, rho, nu, kc, nn, m in rows:
        assert O.counts(int(nB), float(rho), float(nu)) == (int(kc), int(nn), int(m)), rows


def test_counts_reject_bad_ratios():
    for rho, nu in [(0.0, 0.1), (1.1, 0.0), (0.5, -0.1), (0.5, 1.0)]:
        with pytest.raises(ValueError):
            O.counts(16, rho, nu)


# ------------------------------------------------------------------ step 1: smoothing mean
def test_channel_mean_close_to_fp64_mean():
    q, k, v = make_random_qkv(2, 3, 1000, seed=1)
    kf = f32(k)
    mu = O.channel_mean(kf)
    ref = kf.astype(np.float64).mean(axis=2)
    # fp32 summation of N terms: error below N * eps * max|k|.
    bound = 1000 * 2 ** -23 * np.abs(kf).max()
    assert mu.dtype == np.float32
    assert np.abs(mu - ref).max() <= bound


def test_channel_mean_exact_on_dyadic_grid():
    rng = np.random.default_rng(3)
    kf = (rng.integers(-512, 512, size=(1, 2, 1024, 128)) / 64.0).astype(np.float32)
    mu = O.channel_mean(kf)
    # every partial sum is a multiple of 1/64 below 2^24/64, so the sum is exact and
    # N = 1024 is a power of two: the mean is exactly representable.
    np.testing.assert_array_equal(mu, kf.astype(np.float64).mean(axis=2).astype(np.float32))


# ------------------------------------------------------------------ step 3: quantization
def test_quantize_round_half_even_closed_form():
    # One 64-token block, d = 128; the largest |x| is 127 so s = 127/127 = 1 exactly and
    # x8 = rint(x) with ties to even.
    x = np.zeros((1, 1, 64, 128), dtype=np.float32)
    vals = [127.0, 0.5, 1.5, 2.5, -2.5, -63.5, 126.5, -0.5, 3.25, -127.0]
    want = [127, 0, 2, 2, -2, -64, 126, 0, 3, -127]
    x[0, 0, 0, :len(vals)] = vals
    x8, s = O.quantize_blocks(x, 64)
    assert s[0, 0, 0] == np.float32(1.0)
    assert list(x8[0, 0, 0, :len(vals)]) == want
    assert (x8[0, 0, 1:] == 0).all()


def test_quantize_scale_and_error_bound():
    q, k, v = make_random_qkv(1, 2, 300, seed=2)
    x = f32(q) * np.float32(0.37)
    x[0, 1, 64:128] = 0.0  # an all-zero block
    x8, s = O.quantize_blocks(x, 300)
    nB = 5
    assert x8.shape == (1, 2, nB * 64, 128)
    assert s[0, 1, 1] == 0 and (x8[0, 1, 64:128] == 0).all()
    assert (x8[:, :, 300:] == 0).all()  # padded rows
    for hh in range(2):
        for j in range(nB):
            lo, hi = j * 64, min(300, j * 64 + 64)
            blk = x[0, hh, lo:hi].astype(np.float64)
            a = np.abs(blk).max()
            assert s[0, hh, j] == np.float32(np.float32(a) / np.float32(127))
            if a == 0:
                continue
            codes = x8[0, hh, lo:hi].astype(np.float64)
            assert np.abs(codes).max() == 127
            assert np.abs(codes).max() <= 127 and codes.min() >= -127
            err = np.abs(blk - s[0, hh, j] * codes)
            # rint contributes 1/2; the fl32 quotient x/s (|x/s| <= 127 + tiny) adds at
            # most 128 * 2^-24, both in units of s.
            assert err.max() <= s[0, hh, j] * (0.5 + 128 * 2 ** -24)


def test_block_means_close_to_numpy():
    q, k, v = make_random_qkv(1, 2, 200, seed=4)
    x = f32(q)
    m = O.block_means(x, 200)
    for j in range(4):
        lo, hi = j * 64, min(200, j * 64 + 64)
        ref = x[:, :, lo:hi].astype(np.float64).mean(axis=2)
        assert np.abs(m[:, :, j] - ref).max() <= 64 * 2 ** -23 * np.abs(x).max()


# ------------------------------------------------------------------ step 4: selection
def _rn32(x):
    """Round an exact rational to the nearest float32, ties to even (normal and subnormal)."""
    from fractions import Fraction
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    q = max(e, -126) - 23
    m = x / Fraction(2) ** q
    n = m.numerator // m.denominator
    r = m - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(float(sign * n * Fraction(2) ** q))


def test_fma32_is_correctly_rounded():
    # The block logits are a chain of fp32 fused multiply-adds: fl32(a*b + c), one rounding.
    # Checked against exact rational arithmetic on random and cancelling operands, and on a
    # case where rounding a*b + c to float64 first and then to float32 (double rounding)
    # gives the wrong answer: a*b + c = 1 + 3*2^-24 - 2^-70 lies just below a float32
    # midpoint, its float64 rounding lands on the midpoint, and ties-to-even then rounds up.
    from fractions import Fraction
    rng = np.random.default_rng(1)
    n = 3000
    a = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    b = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    p32 = (a.astype(np.float64) * b).astype(np.float32)
    c = np.where(rng.random(n) < 0.5, (-p32 * (1 + rng.integers(-3, 4, n) * 2.0 ** -23)).astype(np.float32),
                 (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32))
    a = np.append(a, np.float32(1 + 2.0 ** -23))
    b = np.append(b, np.float32(2.0 ** -24 * (1 - 2.0 ** -23)))
    c = np.append(c, np.float32(1 + 2.0 ** -23))
    exact = np.array([_rn32(Fraction(float(x)) * Fraction(float(y)) + Fraction(float(z)))
                      for x, y, z in zip(a, b, c)], dtype=np.float32)
    np.testing.assert_array_equal(O.fma32(a, b, c).view(np.uint32), exact.view(np.uint32))
    naive = (a.astype(np.float64) * b + c).astype(np.float32)
    assert naive[-1] != exact[-1]  # the planted case separates the two


def test_logits_close_to_fp64_dot():
    rng = np.random.default_rng(5)
    qb = rng.normal(size=(1, 2, 9, 128)).astype(np.float32)
    kb = rng.normal(size=(1, 2, 7, 128)).astype(np.float32)
    ell = O.block_logits(qb, kb)
    ref = np.einsum("bhic,bhjc->bhij", qb.astype(np.float64), kb.astype(np.float64))
    bound = 128 * 2 ** -22 * np.einsum("bhic,bhjc->bhij", np.abs(qb), np.abs(kb))
    assert ell.dtype == np.float32 and (np.abs(ell - ref) <= bound).all()


def test_select_partition_and_counts():
    q, k, v = make_qkv(1, 2, (4, 16, 16), seed=0)
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
    nB = 16
    assert (sel.k_c, sel.n_neg, sel.m) == (4, 4, 8)
    assert sel.crit.shape == (1, 2, nB, 4) and sel.marg.shape == (1, 2, nB, 8)
    for hh in range(2):
        for i in range(nB):
            c, mg, ng = sel.crit[0, hh, i], sel.marg[0, hh, i], sel.neg[0, hh, i]
            allb = np.concatenate([c, mg, ng])
            assert sorted(allb.tolist()) == list(range(nB))       # disjoint and covering
            for lst in (c, mg, ng):
                assert (np.diff(lst) > 0).all()                   # ascending
            # every critical logit >= every marginal >= every negligible
            e = sel.logits[0, hh, i]
            assert e[c].min() >= e[mg].max() >= e[ng].max() or sel.m == 0


def test_select_order_matches_stable_argsort():
    rng = np.random.default_rng(6)
    qb = rng.normal(size=(2, 3, 20, 128)).astype(np.float32)
    kb = rng.normal(size=(2, 3, 20, 128)).astype(np.float32)
    # force exact ties in a few places: duplicate key blocks
    kb[:, :, 5] = kb[:, :, 2]
    kb[:, :, 17] = kb[:, :, 2]
    sel = O.select(qb, kb, 0.3, 0.3)
    for idx in np.ndindex(2, 3, 20):
        order = np.argsort(-sel.logits[idx].astype(np.float64), kind="stable")
        np.testing.assert_array_equal(sel.crit[idx], np.sort(order[:sel.k_c]))
        np.testing.assert_array_equal(sel.neg[idx], np.sort(order[20 - sel.n_neg:]))


def test_select_ties_go_to_lower_index():
    # Every key block a copy of the first: all logits in a row are equal, so the
    # critical set is {0..k_c-1} and the negligible set is {nB-n_neg..nB-1}.
    q, k, v = make_random_qkv(1, 2, 640, seed=7)
    kf = f32(k)
    kf[:, :, 64:] = np.tile(kf[:, :, :64], (1, 1, 9, 1))
    prep = O.prepare(f32(q), kf)
    sel = O.select(prep.q_bar, prep.k_bar, 0.3, 0.3)
    k_c, n_neg, m = sel.k_c, sel.n_neg, sel.m
    assert (k_c, n_neg, m) == (3, 3, 4)
    for idx in np.ndindex(1, 2, 10):
        assert (sel.logits[idx] == sel.logits[idx][0]).all()
        assert sel.crit[idx].tolist() == [0, 1, 2]
        assert sel.marg[idx].tolist() == [3, 4, 5, 6]
        assert sel.neg[idx].tolist() == [7, 8, 9]


def test_ranking_by_logit_equals_ranking_by_sblk():
    # Ranking by the fp32 S_blk (stable: ties to the lower index) gives the logit lists at
    # both class boundaries except on near-tie rows, where fp32 S_blk leaves the order open.
    for seed, grid in ((1, (4, 16, 16)), (2, (6, 20, 24))):
        q, k, v = make_qkv(1, 2, grid, seed=seed)
        prep = O.prepare(f32(q), f32(k))
        sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
        p = sel.s_blk()
        nB = p.shape[-1]
        assert np.abs(p.astype(np.float64).sum(-1) - 1.0).max() <= nB * 2.0 ** -23
        ties = sel.near_ties(1e-5)
        for idx in np.ndindex(*p.shape[:-1]):
            order = np.argsort(-p[idx], kind="stable")
            same = (np.array_equal(np.sort(order[:sel.k_c]), sel.crit[idx]) and
                    np.array_equal(np.sort(order[nB - sel.n_neg:]), sel.neg[idx]))
            assert same or ties[idx], idx


# ------------------------------------------------------------------ steps 5-7
def test_phi_matches_torch_elu_plus_one():
    x = np.linspace(-30, 30, 2001)
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    # torch forms elu(x) + 1 as (exp(x) - 1) + 1, which loses relative accuracy for
    # very negative x; compare absolutely there (the values are below 1).
    np.testing.assert_allclose(O.phi(x), ref, rtol=1e-15, atol=2e-16)
    np.testing.assert_allclose(O.phi(x[x < 0]), np.exp(x[x < 0]), rtol=1e-15)


@pytest.mark.parametrize("N", [64, 100, 256])
def test_dense_unquantized_equals_sdpa(N):
    q, k, v = make_random_qkv(1, 2, N, seed=N)
    qf, kf, vf = f32(q), f32(k), f32(v)
    c_s = O.softmax_scale(128)
    out, prep, sel = O.sagesla(qf, kf, vf, 1.0, 0.0, quant=False, exact=True)
    assert sel.m == 0 and sel.k_c == prep.n_blocks
    ref = sdpa64(qf, kf, vf, c_s)
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()


def _python_attention(q, k, v, scale):
    """Pure-Python softmax attention (tiny inputs): the textbook formula, loop by loop."""
    N, d = len(q), len(q[0])
    out = []
    for t in range(N):
        s = [sum(q[t][c] * k[u][c] for c in range(d)) * scale for u in range(N)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        out.append([sum(e[u] * v[u][c] for u in range(N)) / tot for c in range(len(v[0]))])
    return out


def test_dense_unquantized_bruteforce_python_small_block():
    # b = 2 tokens per block, d = 3, N = 5 (three blocks, the last one ragged).
    rng = np.random.default_rng(8)
    q = rng.normal(size=(1, 1, 5, 3))
    k = rng.normal(size=(1, 1, 5, 3)) + 3.0
    v = rng.normal(size=(1, 1, 5, 3))
    prep = O.prepare(q, k, v, c_s=0.5, b=2, exact=True)
    sel = O.select(prep.q_bar, prep.k_bar, 1.0, 0.0)
    out = O.forward(prep, v, sel, quant=False)
    ref = _python_attention(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(),
                            float(np.float32(0.5)))
    np.testing.assert_allclose(out[0, 0], np.array(ref), rtol=1e-12, atol=1e-12)


def test_ragged_padding_excluded():
    # N = 100: the second block holds 36 real tokens; padded keys must carry no weight.
    q, k, v = make_random_qkv(1, 1, 100, seed=9)
    qf, kf, vf = f32(q), f32(k), f32(v)
    out, prep, sel = O.sagesla(qf, kf, vf, 1.0, 0.0, quant=False, exact=True)
    ref = sdpa64(qf, kf, vf, O.softmax_scale(128))
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()
    assert out.shape == (1, 1, 100, 128)


def test_k_shift_invariance_exact_mode():
    q, k, v = make_random_qkv(1, 2, 192, seed=10)
    qf, kf, vf = f32(q), f32(k), f32(v)
    shift = np.random.default_rng(11).normal(size=(1, 2, 1, 128)) * 5
    o1, _, _ = O.sagesla(qf, kf, vf, 1.0, 0.0, quant=False, exact=True)
    o2, _, _ = O.sagesla(qf, kf + shift, vf, 1.0, 0.0, quant=False, exact=True)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()
    # and it is the same as attention on the unshifted K (full softmax is K-shift free)
    ref = sdpa64(qf, kf + shift, vf, O.softmax_scale(128))
    assert np.abs(o2 - ref).max() <= 1e-12 * np.abs(ref).max()


def test_k_shift_invariance_bitexact_full_method():
    # Dyadic inputs, N = 1024: mu(K + c) = mu(K) + c exactly, so K~ and everything
    # downstream (INT8 codes, scales, lists, output) are bit-identical.
    rng = np.random.default_rng(12)
    shape = (1, 2, 1024, 128)
    qf = (rng.integers(-256, 256, size=shape) / 64.0).astype(np.float32)
    kf = (rng.integers(-256, 256, size=shape) / 64.0).astype(np.float32)
    vf = rng.normal(size=shape).astype(np.float32)
    c = (rng.integers(-512, 512, size=(1, 2, 1, 128)) / 64.0).astype(np.float32)
    o1, p1, s1 = O.sagesla(qf, kf, vf, 0.25, 0.25)
    o2, p2, s2 = O.sagesla(qf, kf + c, vf, 0.25, 0.25)
    np.testing.assert_array_equal(p1.k_t, p2.k_t)
    np.testing.assert_array_equal(p1.k8, p2.k8)
    np.testing.assert_array_equal(s1.crit, s2.crit)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(p2.k_mean, p1.k_mean + c[:, :, 0])


def test_softmax_rows_sum_to_one():
    q, k, v = make_qkv(1, 2, (4, 16, 16), seed=0)
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
    _, _, _, rs = O.forward(prep, f32(v), sel, return_parts=True)
    np.testing.assert_allclose(rs, 1.0, rtol=0, atol=1e-12)


def _block_tokens(blocks, N, b=64):
    return np.concatenate([np.arange(j * b, min(N, j * b + b)) for j in blocks])


def test_closed_form_zero_queries():
    # Q = 0: every logit is 0 (ties -> critical = first k_c blocks), every INT8 score is
    # 0 (uniform softmax over the critical tokens, P = 1 exactly in bf16), phi(Q~) = 1.
    # So O = mean_crit(V) + sum_marg w_u V_u / sum_marg w_u with w_u = sum_c phi(K~_u[c]).
    q, k, v = make_random_qkv(1, 1, 1000, seed=13)
    qf = np.zeros_like(f32(q))
    kf, vf = f32(k), f32(v)
    out, prep, sel = O.sagesla(qf, kf, vf, 0.25, 0.25)
    nB = 16
    k_c, n_neg, m = O.counts(nB, 0.25, 0.25)
    crit_tok = _block_tokens(range(k_c), 1000)
    marg_tok = _block_tokens(range(k_c, nB - n_neg), 1000)
    kt = prep.k_t[0, 0].astype(np.float64)
    w = O.phi(kt[marg_tok]).sum(axis=1)
    want = vf[0, 0, crit_tok].astype(np.float64).mean(axis=0) + \
        (w[:, None] * vf[0, 0, marg_tok]).sum(axis=0) / w.sum()
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(want, (1000, 128)),
                               rtol=1e-11, atol=1e-12)
    # the smoothing really is applied: K~ has (near) zero channel means
    assert np.abs(kt.mean(axis=0)).max() < 1e-4


def test_closed_form_zero_keys():
    # K = 0: mu = 0, K~ = 0, all logits 0, all scores 0, phi(K~) = 1 everywhere:
    # O = mean_crit(V) + mean_marg(V) for every query, whatever Q is.
    q, k, v = make_random_qkv(1, 1, 1000, seed=14)
    qf, vf = f32(q), f32(v)
    out, prep, sel = O.sagesla(qf, np.zeros_like(qf), vf, 0.25, 0.25)
    k_c, n_neg, m = O.counts(16, 0.25, 0.25)
    want = vf[0, 0, _block_tokens(range(k_c), 1000)].astype(np.float64).mean(0) + \
        vf[0, 0, _block_tokens(range(k_c, 16 - n_neg), 1000)].astype(np.float64).mean(0)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(want, (1000, 128)),
                               rtol=1e-11, atol=1e-12)


def test_linear_branch_matches_token_level_bruteforce():
    # O_l[t] as a similarity-weighted average over the marginal tokens, with similarity
    # phi(q_t) . phi(k_u), summed token by token (no block states).
    q, k, v = make_qkv(1, 1, (2, 8, 16), seed=2)  # N = 256, nB = 4
    qf, kf, vf = f32(q), f32(k), f32(v)
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
    assert sel.m == 2
    _, _, Ol, _ = O.forward(prep, vf, sel, return_parts=True)
    pq = O.phi(prep.q_t[0, 0])
    pk = O.phi(prep.k_t[0, 0])
    for t in range(0, 256, 7):
        toks = _block_tokens(sel.marg[0, 0, t // 64], 256)
        w = np.array([pq[t] @ pk[u] for u in toks])
        want = (w[:, None] * vf[0, 0, toks].astype(np.float64)).sum(0) / w.sum()
        np.testing.assert_allclose(Ol[0, 0, t], want, rtol=1e-12, atol=1e-13)


def test_outputs_are_convex_combinations():
    q, k, v = make_qkv(1, 2, (4, 16, 16), seed=3)
    qf, kf, vf = f32(q), f32(k), f32(v)
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
    _, Os, Ol, _ = O.forward(prep, vf, sel, return_parts=True)
    for hh in range(2):
        for i in range(16):
            ct = _block_tokens(sel.crit[0, hh, i], 1024)
            mt = _block_tokens(sel.marg[0, hh, i], 1024)
            rows = slice(i * 64, i * 64 + 64)
            vc, vm = vf[0, hh, ct], vf[0, hh, mt]
            # bf16(P) over unrounded l: slack of 2^-8 relative to max|V|
            slack = 2 ** -8 * np.abs(vc).max()
            assert (Os[0, hh, rows] <= vc.max(0) + slack).all()
            assert (Os[0, hh, rows] >= vc.min(0) - slack).all()
            assert (Ol[0, hh, rows] <= vm.max(0) + 1e-12).all()
            assert (Ol[0, hh, rows] >= vm.min(0) - 1e-12).all()


def test_quantized_path_close_to_unquantized_dense():
    # Dense SageAttention path (rho = 1, nu = 0): INT8 QK^T + bf16 P against fp64
    # full attention of the bf16 inputs.
    q, k, v = make_qkv(1, 2, (4, 16, 16), seed=5)
    qf, kf, vf = f32(q), f32(k), f32(v)
    out, prep, sel = O.sagesla(qf, kf, vf, 1.0, 0.0)
    ref = sdpa64(qf, kf, vf, O.softmax_scale(128))
    assert cos(out, ref) >= 0.99


def test_no_marginal_blocks_gives_zero_linear_term():
    q, k, v = make_random_qkv(1, 1, 256, seed=15)
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, 0.5, 0.5)
    assert sel.m == 0
    _, Os, Ol, _ = O.forward(prep, f32(v), sel, return_parts=True)
    assert (Ol == 0).all()


# ---------------------------------------------------------------- S_blk in fp32, near ties
def _sel_from_logits(logit_rows, rho, nu):
    """A selection whose block logits are exactly the given values: q_bar = e_0 and
    k_bar[j] = logit_j e_0, so each fused multiply-add chain returns logit_j unrounded."""
    L = np.asarray(logit_rows, dtype=np.float32)
    nQ, nK = L.shape
    d = 4
    qb = np.zeros((1, 1, nQ, d), dtype=np.float32)
    qb[..., 0] = 1.0
    kb = np.zeros((1, 1, nK, d), dtype=np.float32)
    kb[0, 0, :, 0] = L[0]
    sels = []
    for r in range(nQ):
        kb[0, 0, :, 0] = L[r]
        sels.append(O.select(qb[:, :, r:r + 1], kb, rho, nu))
    return sels


def test_s_blk_is_an_fp32_softmax():
    sel = _sel_from_logits([[3.0, 1.0, 0.5, -2.0, 0.0, 1.5, -1.0, 2.0]], 0.25, 0.25)[0]
    p = sel.s_blk()
    assert p.dtype == np.float32
    x = sel.logits[0, 0, 0].astype(np.float64)
    ref = np.exp(x - x.max()) / np.exp(x - x.max()).sum()
    assert np.abs(p[0, 0, 0] - ref).max() <= 8 * 2.0 ** -24  # a few fp32 roundings
    assert abs(float(p.astype(np.float64).sum()) - 1.0) <= 8 * 2.0 ** -24


def test_near_ties_at_both_boundaries():
    # nB = 8, rho = 0.25 -> k_c = 2, nu = 0.25 -> n_neg = 2: boundaries after positions 2 and 6
    apart = [5.0, 4.0, 3.0, 2.0, 1.0, 0.0, -1.0, -2.0]
    sep, = _sel_from_logits([apart], 0.25, 0.25)
    assert not sep.near_ties().any()
    # equal logits across the critical boundary: a tie the logit order breaks by index
    tie_c, = _sel_from_logits([[5.0, 4.0, 4.0, 2.0, 1.0, 0.0, -1.0, -2.0]], 0.25, 0.25)
    assert tie_c.near_ties().all()
    assert tie_c.crit[0, 0, 0].tolist() == [0, 1]  # the lower index of the tied pair is critical
    # logits 1e-7 apart at the negligible boundary: distinct logits, fp32 S_blk within 1e-5
    close, = _sel_from_logits([[5.0, 4.0, 3.0, 2.0, 1.0, -1.0, -1.0000001, -2.0]], 0.25, 0.25)
    assert close.logits[0, 0, 0, 5] > close.logits[0, 0, 0, 6]
    assert close.near_ties().all()
    # far below the row max fp32 S_blk underflows to 0 for both neighbours: still ranked by logit
    under, = _sel_from_logits([[0.0, -1.0, -2.0, -3.0, -4.0, -300.0, -301.0, -302.0]], 0.25, 0.25)
    assert under.s_blk()[0, 0, 0, 5] == 0.0 and under.s_blk()[0, 0, 0, 6] == 0.0
    assert under.near_ties().all()
    assert under.neg[0, 0, 0].tolist() == [6, 7]  # -301 and -302, the two smallest logits


def test_near_tie_tally_on_the_480p_sample():
    # The tally the method's fp32 S_blk leaves open on two heads of the 480p workload (seed 0):
    # rows where the blocks on either side of a class boundary are within 1e-5 relative.
    from quantized_block_sparse_b200.inputs import make_qkv
    q, k, _ = make_qkv(1, 2, (21, 30, 52), seed=0)
    prep = O.prepare(q.float().numpy(), k.float().numpy())
    sel = O.select(prep.q_bar, prep.k_bar, 0.10, 0.45)
    ties = sel.near_ties(1e-5)
    assert ties.shape == (1, 2, 512)
    assert int(ties.sum()) == 30  # of 1024 rows; none is an exact fp32 tie
