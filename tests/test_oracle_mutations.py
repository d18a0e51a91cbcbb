"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

Each mutation replaces one function of the oracle module for the duration of one test;
the pin tests are then re-run and must fail.
"""
import numpy as np
import pytest

import oracle.sagesla_oracle as S
import tests.test_oracle_pins as pins


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_mutation_linear_state_transposed(monkeypatch):
    orig = S.linear_states

    def transposed(k_t, v, N, b=S.BLOCK):
        h, z = orig(k_t, v, N, b)
        return np.swapaxes(h, 1, 2), z

    monkeypatch.setattr(S, "linear_states", transposed)
    assert _fails(pins.test_linear_branch_matches_token_level_bruteforce)


def test_mutation_phi_without_plus_one(monkeypatch):
    monkeypatch.setattr(S, "phi", lambda x: np.where(np.asarray(x) > 0, x, np.expm1(np.minimum(x, 0))))
    with np.errstate(all="ignore"):
        assert _fails(pins.test_linear_branch_matches_token_level_bruteforce)


def test_mutation_ties_to_higher_index(monkeypatch):
    def select_high_first(q_bar, k_bar, rho, nu):
        ell = S.block_logits(q_bar, k_bar)
        nK = ell.shape[-1]
        k_c, n_neg, m = S.counts(nK, rho, nu)
        jj = np.broadcast_to(np.arange(nK), ell.shape)
        order = np.lexsort((-jj, -ell.astype(np.float64)), axis=-1)
        crit = np.sort(order[..., :k_c], axis=-1).astype(np.int32)
        marg = np.sort(order[..., k_c:nK - n_neg], axis=-1).astype(np.int32)
        neg = np.sort(order[..., nK - n_neg:], axis=-1).astype(np.int32)
        return S.Selection(k_c, n_neg, m, ell, order, crit, marg, neg)

    monkeypatch.setattr(pins.O, "select", select_high_first)
    assert _fails(pins.test_select_ties_go_to_lower_index)


def test_mutation_mean_over_channels(monkeypatch):
    def wrong_mean(k, b=S.BLOCK):
        kf = k.astype(np.float32)
        return kf.mean(axis=3)[:, :, : kf.shape[3]].astype(np.float32)

    monkeypatch.setattr(S, "channel_mean", wrong_mean)
    assert _fails(pins.test_k_shift_invariance_bitexact_full_method)


def test_mutation_key_scale_dropped(monkeypatch):
    orig = S.prepare

    def no_kscale(*a, **kw):
        p = orig(*a, **kw)
        p.k_scale = np.ones_like(p.k_scale)
        return p

    monkeypatch.setattr(S, "prepare", no_kscale)
    monkeypatch.setattr(pins.O, "sagesla", S.sagesla)
    assert _fails(pins.test_quantized_path_close_to_unquantized_dense)


def test_mutation_padding_not_masked(monkeypatch):
    orig = S.forward

    def no_mask(prep, v, sel, **kw):
        # pretend every block is full: padded keys (zero K~, zero V) enter the softmax
        N = prep.N
        nB = prep.n_blocks
        pad = nB * prep.block
        qt = np.zeros(prep.q_t.shape[:2] + (pad, prep.q_t.shape[3]), prep.q_t.dtype)
        kt = np.zeros_like(qt)
        qt[:, :, :N] = prep.q_t
        kt[:, :, :N] = prep.k_t
        vp = np.zeros(qt.shape)
        vp[:, :, :N] = v
        p2 = S.Prepared(pad, prep.block, qt, kt, prep.k_mean, prep.q8, prep.k8,
                        prep.q_scale, prep.k_scale, prep.q_bar, prep.k_bar)
        return orig(p2, vp, sel, **kw)[:, :, :N]

    monkeypatch.setattr(S, "forward", no_mask)
    monkeypatch.setattr(pins.O, "sagesla", S.sagesla)
    assert _fails(pins.test_ragged_padding_excluded)


def test_mutation_rint_truncates(monkeypatch):
    monkeypatch.setattr(S.np, "rint", np.trunc)
    try:
        assert _fails(pins.test_quantize_round_half_even_closed_form)
    finally:
        monkeypatch.undo()


def test_mutation_scale_over_128(monkeypatch):
    orig = S.quantize_blocks

    def over_128(X, N, b=S.BLOCK):
        x8, s = orig(X, N, b)
        s128 = (s * np.float32(127) / np.float32(128)).astype(np.float32)
        return x8, s128

    monkeypatch.setattr(S, "quantize_blocks", over_128)
    monkeypatch.setattr(pins.O, "quantize_blocks", over_128)
    assert _fails(pins.test_quantize_round_half_even_closed_form)


def test_mutation_softmax_scale_folded_twice(monkeypatch):
    orig = S.prepare

    def twice(q, k, v=None, c_s=None, b=S.BLOCK, smooth=True, exact=False):
        cs = S.softmax_scale(np.asarray(q).shape[-1]) if c_s is None else c_s
        return orig(np.asarray(q) * float(cs), k, v, c_s, b, smooth, exact)

    monkeypatch.setattr(S, "prepare", twice)
    assert _fails(lambda: pins.test_dense_unquantized_equals_sdpa(64))


def test_mutation_linear_branch_on_unsmoothed_keys(monkeypatch):
    orig = S.prepare

    def unsmoothed(q, k, v=None, c_s=None, b=S.BLOCK, smooth=True, exact=False):
        p = orig(q, k, v, c_s, b, smooth, exact)
        p.k_t = np.asarray(k, dtype=p.k_t.dtype)  # phi(K) instead of phi(K~) downstream
        return p

    monkeypatch.setattr(S, "prepare", unsmoothed)
    assert _fails(pins.test_k_shift_invariance_bitexact_full_method)


def test_mutation_negligible_ties_to_lower_index(monkeypatch):
    orig = S.select

    def low_negligible(q_bar, k_bar, rho, nu):
        sel = orig(q_bar, k_bar, rho, nu)
        ell = sel.logits
        nK = ell.shape[-1]
        jj = np.broadcast_to(np.arange(nK), ell.shape)
        low_first = np.lexsort((jj, ell.astype(np.float64)), axis=-1)  # lowest logit, lower index
        neg = np.sort(low_first[..., :sel.n_neg], axis=-1).astype(np.int32)
        return S.Selection(sel.k_c, sel.n_neg, sel.m, ell, sel.rank, sel.crit, sel.marg, neg)

    monkeypatch.setattr(pins.O, "select", low_negligible)
    assert _fails(pins.test_select_ties_go_to_lower_index)
