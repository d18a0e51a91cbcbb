"""Pins for the SageSLA backward oracle (oracle/sla_backward_oracle.py), CPU only.

The gradients come from autograd over a dense restatement of the forward, so the pins
check it against independent things: the forward against the pinned numpy oracle's
unquantized path, the gradients against central finite differences, and dK against the
method's invariance to a per-channel constant added to K. Planted mistakes must fail them.
"""
import numpy as np
import torch

import oracle as O
import oracle.sla_backward_oracle as G


def _case(N=200, d=16, rho=0.5, nu=0.25, seed=0, H=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, N, d))
    k = rng.standard_normal((1, H, N, d)) + rng.standard_normal((1, H, 1, d)) * 2
    v = rng.standard_normal((1, H, N, d))
    do = rng.standard_normal((1, H, N, d))
    prep = O.prepare(q, k, exact=True)
    sel = O.select(prep.q_bar, prep.k_bar, rho, nu)
    return q, k, v, do, prep, sel


def _loss(q, k, v, do, sel):
    out, _ = G.forward_backward(q, k, v, do, sel)
    return float((out * do).sum())


def test_forward_matches_numpy_oracle_unquantized():
    for (N, rho, nu) in [(200, 0.5, 0.25), (129, 1.0, 0.0), (320, 0.2, 0.2)]:
        q, k, v, do, prep, sel = _case(N=N, rho=rho, nu=nu)
        ref = O.forward(prep, v, sel, quant=False)
        out, _ = G.forward_backward(q, k, v, do, sel)
        np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_gradients_match_central_differences():
    q, k, v, do, _, sel = _case(N=150, d=8, rho=0.5, nu=0.3, seed=1)
    _, (dq, dk, dv) = G.forward_backward(q, k, v, do, sel)
    rng = np.random.default_rng(5)
    eps = 1e-5
    for _ in range(3):
        uq, uk, uv = (rng.standard_normal(q.shape) for _ in range(3))
        lp = _loss(q + eps * uq, k + eps * uk, v + eps * uv, do, sel)
        lm = _loss(q - eps * uq, k - eps * uk, v - eps * uv, do, sel)
        fd = (lp - lm) / (2 * eps)
        an = float((dq * uq).sum() + (dk * uk).sum() + (dv * uv).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)


def test_dk_sums_to_zero_over_tokens():
    # O is unchanged by K + 1 c^T (smoothing removes it), so dO/dK has no component along it
    for (rho, nu) in [(0.5, 0.25), (1.0, 0.0), (0.25, 0.0)]:
        q, k, v, do, _, sel = _case(N=256, rho=rho, nu=nu, seed=2)
        _, (_, dk, _) = G.forward_backward(q, k, v, do, sel)
        colsum = np.abs(dk.sum(axis=2)).max()
        assert colsum <= 1e-10 * np.abs(dk).max(), colsum
        assert np.abs(dk).max() > 1e-3  # not trivially zero


def test_dv_of_softmax_only_rows():
    # rho = 1: every key block critical, no linear branch: dV = P^T dO with P the softmax
    # of the fold-scaled scores over all real tokens
    q, k, v, do, prep, sel = _case(N=130, rho=1.0, nu=0.0, seed=3, H=1)
    _, (_, _, dv) = G.forward_backward(q, k, v, do, sel)
    s = prep.q_t[0, 0] @ prep.k_t[0, 0].T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(dv[0, 0], p.T @ do[0, 0], rtol=1e-10, atol=1e-12)


# ---- planted mistakes

def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_mutation_mean_detached(monkeypatch):
    monkeypatch.setattr(G, "head_forward", _detached_forward)
    assert _fails(test_dk_sums_to_zero_over_tokens)


def _detached_forward(q, k, v, crit_rows, marg_rows, c_s, b):
    N = q.shape[0]
    nB = -(-N // b)
    qt = q * c_s
    kt = k - k.mean(dim=0, keepdim=True).detach()  # the mistake: mu treated as a constant
    crit = G._token_mask(crit_rows, nB, N, b)
    o = torch.softmax((qt @ kt.T).masked_fill(~crit, float("-inf")), dim=1) @ v
    if marg_rows.shape[1]:
        a = (G._phi(qt) @ G._phi(kt).T) * G._token_mask(marg_rows, nB, N, b)
        den = a.sum(dim=1, keepdim=True)
        o = o + (a @ v) / torch.where(den > 0, den, torch.ones_like(den))
    return o


def test_mutation_linear_branch_unnormalised(monkeypatch):
    def unnormalised(q, k, v, crit_rows, marg_rows, c_s, b=O.BLOCK):
        N = q.shape[0]
        nB = -(-N // b)
        qt, kt = q * c_s, k - k.mean(dim=0, keepdim=True)
        crit = G._token_mask(crit_rows, nB, N, b)
        o = torch.softmax((qt @ kt.T).masked_fill(~crit, float("-inf")), dim=1) @ v
        if marg_rows.shape[1]:
            a = (G._phi(qt) @ G._phi(kt).T) * G._token_mask(marg_rows, nB, N, b)
            o = o + a @ v  # the mistake: no division by phi(Q~) . Z
        return o

    monkeypatch.setattr(G, "head_forward", unnormalised)
    assert _fails(test_forward_matches_numpy_oracle_unquantized)
