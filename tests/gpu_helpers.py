"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI, run the
oracle on the same inputs, and compare the way the method requires (bit-exact integers,
scales, means and lists; tolerance on the floating-point output)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from quantized_block_sparse_b200 import sagesla as S

# Output tolerance against the oracle's quantized path: cosine >= 0.9995 and
# max |O - O_ref| <= 2e-2 * max |O_ref|.
COS_MIN = 0.9995
MAXERR_REL = 2e-2
# Cosine reported (and required) against fp64 unquantized attention with the same blocks.
COS_UNQUANT_MIN = 0.99
NEAR_TIE_REL = 1e-5


def ensure_lib():
    import os
    if not os.path.exists(S.LIB_PATH):
        from quantized_block_sparse_b200.build import build
        build()
    return S.lib()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def run_gpu(q, k, v, rho, nu, logits=True, repeat=1):
    """Run prepare, select and forward on cuda:0; return CPU numpy copies."""
    ensure_lib()
    B, H, N, d = q.shape
    qd, kd, vd = (t.cuda().contiguous() for t in (q, k, v))
    eng = S.SageSLA(B, H, N, rho, nu, logits=logits)
    outs = []
    for _ in range(repeat):
        out = eng(qd, kd, vd)
        torch.cuda.synchronize()
        outs.append(out.clone())
    eng.check()
    p, s = eng.prep, eng.sel
    res = dict(
        q8=p.q8.cpu().numpy(), k8=p.k8.cpu().numpy(), q_scale=p.q_scale.cpu().numpy(),
        k_scale=p.k_scale.cpu().numpy(), k_mean=p.k_mean.cpu().numpy(),
        q_bar=p.q_bar.cpu().numpy(), k_bar=p.k_bar.cpu().numpy(),
        h=p.h.float().cpu().numpy(), z=p.z.cpu().numpy(),
        crit=s.crit.cpu().numpy(), marg=s.marg.cpu().numpy()[..., : s.m],
        mask=s.mask.float().cpu().numpy(), k_c=s.k_c, n_neg=s.n_neg, m=s.m,
        logits=None if s.logits is None else s.logits.cpu().numpy(),
        out=outs[-1].float().cpu().numpy(), outs=[o.float().cpu().numpy() for o in outs])
    return res


def run_gpu_select(q, k, v, rho, nu):
    """Run prepare and select only (logits kept); return CPU numpy copies."""
    ensure_lib()
    B, H, N, d = q.shape
    qd, kd, vd = (t.cuda().contiguous() for t in (q, k, v))
    ws = S.alloc_workspace(B, H, N, qd.device)
    p = S.sagesla_prepare(qd, kd, vd, ws)
    s = S.sagesla_select(p.q_bar, p.k_bar, N, rho, nu, logits=True)
    torch.cuda.synchronize()
    S.sagesla_check_status(ws)
    return dict(
        q8=p.q8.cpu().numpy(), k8=p.k8.cpu().numpy(), q_scale=p.q_scale.cpu().numpy(),
        k_scale=p.k_scale.cpu().numpy(), k_mean=p.k_mean.cpu().numpy(),
        q_bar=p.q_bar.cpu().numpy(), k_bar=p.k_bar.cpu().numpy(),
        crit=s.crit.cpu().numpy(), marg=s.marg.cpu().numpy()[..., : s.m],
        mask=s.mask.float().cpu().numpy(), k_c=s.k_c, n_neg=s.n_neg, m=s.m,
        logits=s.logits.cpu().numpy())


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_prepare_bitexact(g, prep, heads=slice(None)):
    np.testing.assert_array_equal(g["q8"][:, heads], prep.q8)
    np.testing.assert_array_equal(g["k8"][:, heads], prep.k8)
    for name in ("q_scale", "k_scale", "k_mean", "q_bar", "k_bar"):
        np.testing.assert_array_equal(bits(g[name][:, heads]), bits(getattr(prep, name)), err_msg=name)


def assert_linear_states_close(g, prep, v, heads_idx, N):
    """h (bf16 output of an fp32-accumulated bf16 MMA) and z against fp64."""
    for (b, h) in heads_idx:
        hh, zz = O.linear_states(prep.k_t[b, h], v[b, h].astype(np.float64), N)
        gh = g["h"][b, h].astype(np.float64)
        gz = g["z"][b, h].astype(np.float64)
        scale = np.abs(hh).max()
        assert np.abs(gh - hh).max() <= 2 ** -6 * scale, "h"
        c = (gh * hh).sum() / np.sqrt((gh * gh).sum() * (hh * hh).sum())
        assert c >= 0.99999, c
        assert np.abs(gz - zz).max() <= 1e-4 * np.abs(zz).max(), "z"


def compare_lists(g, sel, heads=slice(None)):
    """Bit-exact lists; a differing row must be a near-tie at a class boundary.
    Returns the number of near-tie rows."""
    gc, gm = g["crit"][:, heads], g["marg"][:, heads]
    if g["logits"] is not None:
        np.testing.assert_array_equal(bits(g["logits"][:, heads]), bits(sel.logits))
    bad = np.argwhere((gc != sel.crit).any(-1) | ((gm != sel.marg).any(-1) if sel.m else False))
    nB = sel.logits.shape[-1]
    # the bf16 marginal mask: 1 exactly on the marginal blocks, 0 elsewhere and on padding
    gmask = g["mask"][:, heads]
    ok_rows = np.ones(gmask.shape[:-1], dtype=bool)
    ok_rows[tuple(bad.T)] = False
    np.testing.assert_array_equal(gmask[..., :nB][ok_rows], sel.marg_mask()[ok_rows])
    assert not gmask[..., nB:].any()
    near = 0
    ties = sel.near_ties(NEAR_TIE_REL)
    for idx in bad:
        idx = tuple(idx)
        assert ties[idx], f"list mismatch that is not a near-tie at row {idx}"
        near += 1
    return near


def cos(a, b):
    a = a.reshape(-1).astype(np.float64)
    b = b.reshape(-1).astype(np.float64)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def assert_output_close(gout, ref, ref_unq=None):
    m = ~np.isnan(ref)
    a, b = gout[m], ref[m]
    c = cos(a, b)
    err = np.abs(a - b).max()
    assert c >= COS_MIN, f"cos {c}"
    assert err <= MAXERR_REL * np.abs(b).max(), f"max err {err} vs {np.abs(b).max()}"
    out = dict(cos=c, maxerr=float(err), maxref=float(np.abs(b).max()))
    if ref_unq is not None:
        cu = cos(gout[m], ref_unq[m])
        assert cu >= COS_UNQUANT_MIN, f"cos vs unquantized {cu}"
        out["cos_unquant"] = cu
    return out
