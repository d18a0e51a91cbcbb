"""CPU oracle for SageSLA attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this module. The product path (the CUDA library and its Python binding) never
reaches it: it shares no code, table or helper with the CUDA kernels.

What it computes (the method as the pages outline it, made exact):

* "TurboDiffusion Demystified: How It Achieves 100x Faster Video Generation",
  section "Pillar One: Low-Bit Attention Acceleration - SageAttention": attention is
  quantized to INT8 with a smoothing step against outliers.
* same page, section "Pillar Two: Sparse-Linear Attention - SLA": only the most
  important block interactions are computed exactly (about 10% at ``--sla_topk 0.1``,
  section "Hands-On Tutorial"), a light linear-attention term covers the rest, and the
  two stack ("SageSLA").

The exact SageSLA definition this oracle implements, per (batch, head), block b = 64:

1. K is smoothed: K~ = K - mean over the N real tokens, per channel.
2. The softmax scale c_s = fl32(1/sqrt(d)) is folded into Q: Q~ = fl32(Q * c_s).
3. Q~ and K~ are quantized per 64-token block to symmetric INT8:
   s = fl32(max|x| / 127), x8 = clamp(rint(fl32(x / s)), -127, 127) (ties to even).
4. Block logits l_ij = mean(Q~_i) . mean(K~_j) in fp32; S_blk = softmax_j(l).
   Per query-block row the top k_c = ceil(rho * nB) key blocks are critical, the
   bottom n_neg = floor(nu * nB) are negligible, the rest marginal; equal logits
   rank the lower block index first.
5. Critical blocks: exact softmax attention on s = (q8 . k8) * s_q * s_k, with P
   rounded to bf16 before the P.V product.
6. Marginal blocks: linear attention with phi(x) = elu(x) + 1,
   h_j = phi(K~_j)^T V_j, z_j = phi(K~_j)^T 1, H_i = sum_marg h_j, Z_i = sum_marg z_j,
   O_l = phi(Q~)^T H_i / (phi(Q~)^T Z_i)  (0 when the marginal set is empty).
7. O = O_s + O_l; negligible blocks contribute nothing.

Precision: steps 1-4 run in fp32 in the fixed order stated at each function, because
they decide integers (INT8 codes, block lists) that must match bit for bit; steps 5-7
run in fp64 (bf16 rounding of P being part of the method).

Every function is pinned by CPU tests against closed forms, invariances, library
routines (torch SDPA, torch elu, numpy sorts) and brute force on tiny inputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

BLOCK = 64
_F32 = np.float32


# ----------------------------------------------------------------------------------
# Counts (step 4): how many key blocks per row are critical / negligible / marginal.
# ----------------------------------------------------------------------------------
def _near_integer(x: float):
    """Return round(x) if x is within 1e-9 (relative) of an integer, else None.

    rho and nu are decimal ratios (0.1, 0.45, ...); their binary product with nB can
    land a hair above or below an integer (0.3 * 10 = 3.0000000000000004). The count
    is meant for the real product, so such values snap to the integer.
    """
    r = round(x)
    if abs(x - r) <= 1e-9 * max(1.0, abs(x)):
        return int(r)
    return None


def counts(n_blocks: int, rho: float, nu: float):
    """(k_c, n_neg, m) for one query-block row with n_blocks key blocks.

    k_c = ceil(rho * nB) (at least 1), n_neg = floor(nu * nB) capped at nB - k_c,
    m = nB - k_c - n_neg. Requires 0 < rho <= 1, 0 <= nu < 1.
    """
    if not (0.0 < rho <= 1.0) or not (0.0 <= nu < 1.0) or n_blocks < 1:
        raise ValueError("need 0 < rho <= 1, 0 <= nu < 1, n_blocks >= 1")
    xr = rho * n_blocks
    kr = _near_integer(xr)
    k_c = kr if kr is not None else math.ceil(xr)
    k_c = max(1, min(n_blocks, k_c))
    xn = nu * n_blocks
    nr = _near_integer(xn)
    n_neg = nr if nr is not None else math.floor(xn)
    n_neg = max(0, min(n_blocks - k_c, n_neg))
    return k_c, n_neg, n_blocks - k_c - n_neg


def softmax_scale(d: int) -> np.float32:
    """c_s = fl32(1 / sqrt(d)), evaluated once in double precision then rounded."""
    return _F32(1.0 / math.sqrt(float(d)))


# ----------------------------------------------------------------------------------
# Prepare (steps 1-3 and the block means of step 4)
# ----------------------------------------------------------------------------------
@dataclass
class Prepared:
    N: int
    block: int
    q_t: np.ndarray      # Q~ [B,H,N,d]  (fp32; fp64 in exact mode)
    k_t: np.ndarray      # K~ [B,H,N,d]
    k_mean: np.ndarray   # mu [B,H,d] fp32
    q8: np.ndarray       # int8 [B,H,Npad,d], padded rows 0
    k8: np.ndarray
    q_scale: np.ndarray  # fp32 [B,H,nB]
    k_scale: np.ndarray
    q_bar: np.ndarray    # fp32 [B,H,nB,d]
    k_bar: np.ndarray

    @property
    def n_blocks(self) -> int:
        return self.q_scale.shape[-1]


def _valid_mask(N: int, nB: int, b: int) -> np.ndarray:
    """[nB, b] booleans: token j*b + r is a real token (< N)."""
    return (np.arange(nB)[:, None] * b + np.arange(b)[None, :]) < N


def _pad_blocks(X: np.ndarray, nB: int, b: int) -> np.ndarray:
    B, H, N, d = X.shape
    Xp = np.zeros((B, H, nB * b, d), dtype=X.dtype)
    Xp[:, :, :N] = X
    return Xp.reshape(B, H, nB, b, d)


def channel_mean(k: np.ndarray, b: int = BLOCK) -> np.ndarray:
    """Per-channel mean of K over the N real tokens (step 1), fp32, fixed order.

    Order: for every block j, P_j[c] = sum of K[t, c] over the real tokens of block j,
    added one token at a time in increasing t starting from +0.0; then
    T[c] = sum of P_j[c] over j = 0..nB-1 in increasing j starting from +0.0;
    mu[c] = fl32(T[c] / N).
    """
    B, H, N, d = k.shape
    nB = -(-N // b)
    Kb = _pad_blocks(k.astype(_F32), nB, b)
    valid = _valid_mask(N, nB, b)
    P = np.zeros((B, H, nB, d), dtype=_F32)
    for r in range(b):
        vr = valid[:, r][None, None, :, None]
        P = np.where(vr, P + Kb[:, :, :, r, :], P)
    T = np.zeros((B, H, d), dtype=_F32)
    for j in range(nB):
        T = T + P[:, :, j, :]
    return (T / _F32(N)).astype(_F32)


def quantize_blocks(X: np.ndarray, N: int, b: int = BLOCK):
    """Symmetric per-block INT8 quantization (step 3).

    X is fp32 [B,H,N,d]. For each b-token block, over its real tokens and all d
    channels: a = max|x|, s = fl32(a / 127), x8 = clamp(rint(fl32(x / s)), -127, 127)
    with rint rounding half to even; an all-zero block gives s = 0 and x8 = 0.
    Returns (x8 int8 [B,H,nB*b,d] with padded rows 0, s fp32 [B,H,nB]).
    """
    B, H, _, d = X.shape
    nB = -(-N // b)
    Xb = _pad_blocks(X.astype(_F32), nB, b)
    valid = _valid_mask(N, nB, b)[None, None, :, :, None]
    amax = np.where(valid, np.abs(Xb), _F32(0)).max(axis=(3, 4)).astype(_F32)
    s = (amax / _F32(127.0)).astype(_F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (Xb / s[:, :, :, None, None]).astype(_F32)
    y = np.where(s[:, :, :, None, None] > 0, y, _F32(0))
    x8 = np.clip(np.rint(y), -127, 127)
    x8 = np.where(valid, x8, 0).astype(np.int8)
    return x8.reshape(B, H, nB * b, d), s


def block_means(X: np.ndarray, N: int, b: int = BLOCK) -> np.ndarray:
    """Mean over the real tokens of each block (for the step-4 logits), fp32.

    Sum one token at a time in increasing t starting from +0.0, then one fl32 divide
    by the number of real tokens in the block.
    """
    B, H, _, d = X.shape
    nB = -(-N // b)
    Xb = _pad_blocks(X.astype(_F32), nB, b)
    valid = _valid_mask(N, nB, b)
    acc = np.zeros((B, H, nB, d), dtype=_F32)
    for r in range(b):
        vr = valid[:, r][None, None, :, None]
        acc = np.where(vr, acc + Xb[:, :, :, r, :], acc)
    n_valid = valid.sum(axis=1).astype(_F32)
    return (acc / n_valid[None, None, :, None]).astype(_F32)


def prepare(q, k, v=None, c_s=None, b: int = BLOCK, smooth: bool = True,
            exact: bool = False) -> Prepared:
    """Steps 1-3 plus the block means of step 4.

    q, k: float arrays [B,H,N,d] (the bf16 inputs, widened exactly).
    smooth=False skips step 1 (mu = 0). exact=True keeps Q~ and K~ in fp64 (mean in
    fp64) for the unquantized self-checks; INT8 codes are then still produced from
    the fp32-rounded Q~/K~ but are not used by forward(quant=False).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    B, H, N, d = q.shape
    if c_s is None:
        c_s = softmax_scale(d)
    c_s = _F32(c_s)
    if exact:
        qt = q.astype(np.float64) * float(c_s)
        mu64 = k.astype(np.float64).mean(axis=2) if smooth else np.zeros((B, H, d))
        kt = k.astype(np.float64) - mu64[:, :, None, :]
        mu = mu64.astype(_F32)
        qt32, kt32 = qt.astype(_F32), kt.astype(_F32)
    else:
        qt = (q.astype(_F32) * c_s).astype(_F32)
        mu = channel_mean(k, b) if smooth else np.zeros((B, H, d), dtype=_F32)
        kt = (k.astype(_F32) - mu[:, :, None, :]).astype(_F32)
        qt32, kt32 = qt, kt
    q8, sq = quantize_blocks(qt32, N, b)
    k8, sk = quantize_blocks(kt32, N, b)
    qbar = block_means(qt32, N, b)
    kbar = block_means(kt32, N, b)
    return Prepared(N, b, qt, kt, mu, q8, k8, sq, sk, qbar, kbar)


# ----------------------------------------------------------------------------------
# Select (step 4)
# ----------------------------------------------------------------------------------
@dataclass
class Selection:
    k_c: int
    n_neg: int
    m: int
    logits: np.ndarray   # fp32 [B,H,nB,nB]
    rank: np.ndarray     # int [B,H,nB,nB]: position of key block j in row i's order
    crit: np.ndarray     # int32 [B,H,nB,k_c] ascending
    marg: np.ndarray     # int32 [B,H,nB,m] ascending
    neg: np.ndarray      # int32 [B,H,nB,n_neg] ascending

    def s_blk(self) -> np.ndarray:
        """S_blk = softmax_j of the fp32 logits, in fp32 as the method states (max subtracted,
        exp, row sum and divide each rounded to fp32). Reported, not ranked on: the lists
        rank by the logit itself (the refinement of reading A7)."""
        x = self.logits.astype(_F32)
        e = np.exp((x - x.max(axis=-1, keepdims=True)).astype(_F32)).astype(_F32)
        return (e / e.sum(axis=-1, keepdims=True, dtype=_F32)).astype(_F32)

    def near_ties(self, rel: float = 1e-5) -> np.ndarray:
        """bool [B,H,nB]: rows where fp32 S_blk cannot separate the two blocks on either side
        of a class boundary (critical | marginal at position k_c, marginal | negligible at
        nB - n_neg, in the logit order): equal values, or values within `rel` (relative).
        There the method as stated in fp32 leaves the order open and the logit order (which
        breaks such ties) is a refinement; these rows are the near-tie tally."""
        p = self.s_blk().astype(np.float64)
        nB = p.shape[-1]
        order = np.argsort(self.rank, axis=-1)  # position -> block
        ps = np.take_along_axis(p, order, axis=-1)
        out = np.zeros(p.shape[:-1], dtype=bool)
        for pos in (self.k_c, nB - self.n_neg):
            if 0 < pos < nB:
                a, b = ps[..., pos - 1], ps[..., pos]
                out |= (a - b) <= rel * a
        return out

    def marg_mask(self) -> np.ndarray:
        nB = self.logits.shape[-1]
        B, H = self.logits.shape[:2]
        M = np.zeros((B, H, nB, nB), dtype=np.float64)
        if self.m:
            np.put_along_axis(M, self.marg.astype(np.int64), 1.0, axis=-1)
        return M


def fma32(a, b, c) -> np.ndarray:
    """fl32(a*b + c) for float32 a, b, c: one rounding, to nearest even (IEEE fusedMultiplyAdd).

    a*b is exact in float64 (24 + 24 bits). p + c is formed in float64 with round-to-odd:
    the float64 sum s and its exact error e (Knuth's TwoSum) give the odd neighbour of the
    exact value whenever e != 0. A value rounded to odd in a format with at least 2 more
    bits than the target (53 >= 24 + 2) rounds to the target exactly as the exact value
    would (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved
    algorithms using rounding to odd", IEEE Trans. Computers 57(4), 2008), so the final cast
    to float32 is the correctly rounded result.
    """
    p = np.asarray(a, dtype=np.float64) * np.asarray(b, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)
    bits = s.view(np.int64)
    even = (bits & 1) == 0
    fix = (e != 0) & even & np.isfinite(s)
    s_odd = np.where(fix, np.nextafter(s, np.where(e > 0, np.inf, -np.inf)), s)
    return s_odd.astype(_F32)


def block_logits(q_bar: np.ndarray, k_bar: np.ndarray) -> np.ndarray:
    """l_ij = mean(Q~_i) . mean(K~_j) in fp32.

    Fixed order, one fused multiply-add per channel: acc = +0.0; for c = 0..d-1:
    acc = fl32(qbar_i[c] * kbar_j[c] + acc).
    """
    qb = q_bar.astype(_F32)
    kb = k_bar.astype(_F32)
    B, H, nB, d = qb.shape
    acc = np.zeros((B, H, nB, kb.shape[2]), dtype=_F32)
    for c in range(d):
        acc = fma32(qb[:, :, :, None, c], kb[:, :, None, :, c], acc)
    return acc


def select(q_bar, k_bar, rho: float, nu: float) -> Selection:
    """Classify key blocks per query-block row (step 4).

    Rank key blocks by (logit descending, block index ascending): the first k_c are
    critical, the last n_neg negligible, the rest marginal. Ranking on the logit is
    the same as ranking on S_blk = softmax(logit), which is strictly increasing in it.
    """
    ell = block_logits(q_bar, k_bar)
    B, H, nQ, nK = ell.shape
    k_c, n_neg, m = counts(nK, rho, nu)
    jj = np.broadcast_to(np.arange(nK), ell.shape)
    order = np.lexsort((jj, -ell.astype(np.float64)), axis=-1)
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.broadcast_to(np.arange(nK), ell.shape), axis=-1)
    crit = np.sort(order[..., :k_c], axis=-1).astype(np.int32)
    marg = np.sort(order[..., k_c:nK - n_neg], axis=-1).astype(np.int32)
    neg = np.sort(order[..., nK - n_neg:], axis=-1).astype(np.int32)
    return Selection(k_c, n_neg, m, ell, rank, crit, marg, neg)


# ----------------------------------------------------------------------------------
# Forward (steps 5-7)
# ----------------------------------------------------------------------------------
def phi(x: np.ndarray) -> np.ndarray:
    """phi(x) = elu(x) + 1 = x + 1 for x > 0, exp(x) otherwise (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest even) through fp32, returned widened to fp64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def linear_states(k_t: np.ndarray, v: np.ndarray, N: int, b: int = BLOCK):
    """h_j = phi(K~_j)^T V_j  [nB,d,d] and z_j = phi(K~_j)^T 1  [nB,d], one head, fp64.

    Only the real tokens of each block contribute.
    """
    Nk, d = k_t.shape
    nB = -(-N // b)
    h = np.zeros((nB, d, v.shape[1]))
    z = np.zeros((nB, d))
    for j in range(nB):
        lo, hi = j * b, min(N, j * b + b)
        pk = phi(k_t[lo:hi])
        h[j] = pk.T @ v[lo:hi].astype(np.float64)
        z[j] = pk.sum(axis=0)
    return h, z


def forward(prep: Prepared, v, sel: Selection, heads=None, qblocks=None,
            quant: bool = True, return_parts: bool = False):
    """Steps 5-7 for the requested (b, h) heads and query blocks.

    Returns O as fp64 [B,H,N,d]; rows of query blocks not requested are NaN.
    quant=False replaces the INT8 scores by fp64 Q~.K~ and skips the bf16 rounding of
    P (the unquantized reference with the same block selection).
    With return_parts, also returns (O_s, O_l, row_sums) where row_sums holds, per
    computed row, the sum of the normalised softmax weights.
    """
    v = np.asarray(v)
    B, H, N, d = prep.q_t.shape
    b = prep.block
    nB = prep.n_blocks
    if heads is None:
        heads = [(bb, hh) for bb in range(B) for hh in range(H)]
    if qblocks is None:
        qblocks = range(nB)
    qblocks = list(qblocks)
    O = np.full((B, H, N, d), np.nan)
    Os = np.full((B, H, N, d), np.nan) if return_parts else None
    Ol = np.full((B, H, N, d), np.nan) if return_parts else None
    rs = np.full((B, H, N), np.nan) if return_parts else None
    tok_block = np.arange(nB * b) // b
    for (bb, hh) in heads:
        vv = v[bb, hh].astype(np.float64)
        if sel.m > 0:
            h, z = linear_states(prep.k_t[bb, hh], vv, N, b)
            M = sel.marg_mask()[bb, hh]
            Hm = (M @ h.reshape(nB, -1)).reshape(nB, d, -1)
            Zm = M @ z
        for i in qblocks:
            lo, hi = i * b, min(N, i * b + b)
            keys = np.concatenate([np.arange(j * b, min(N, j * b + b))
                                   for j in sel.crit[bb, hh, i]])
            if quant:
                acc = prep.q8[bb, hh, lo:hi].astype(np.float64) @ \
                    prep.k8[bb, hh, keys].astype(np.float64).T
                s = acc * float(prep.q_scale[bb, hh, i]) * \
                    prep.k_scale[bb, hh, tok_block[keys]].astype(np.float64)[None, :]
            else:
                s = prep.q_t[bb, hh, lo:hi].astype(np.float64) @ \
                    prep.k_t[bb, hh, keys].astype(np.float64).T
            mx = s.max(axis=1, keepdims=True)
            p = np.exp(s - mx)
            l = p.sum(axis=1, keepdims=True)
            pv = round_bf16(p) if quant else p
            o_s = (pv @ vv[keys]) / l
            if sel.m > 0:
                pq = phi(prep.q_t[bb, hh, lo:hi])
                o_l = (pq @ Hm[i]) / (pq @ Zm[i])[:, None]
            else:
                o_l = np.zeros_like(o_s)
            O[bb, hh, lo:hi] = o_s + o_l
            if return_parts:
                Os[bb, hh, lo:hi] = o_s
                Ol[bb, hh, lo:hi] = o_l
                rs[bb, hh, lo:hi] = (p / l).sum(axis=1)
    if return_parts:
        return O, Os, Ol, rs
    return O


def sagesla(q, k, v, rho: float, nu: float, c_s=None, heads=None, qblocks=None,
            quant: bool = True, smooth: bool = True, exact: bool = False):
    """Steps 1-7 end to end. Returns (O fp64, Prepared, Selection)."""
    prep = prepare(q, k, v, c_s, smooth=smooth, exact=exact)
    sel = select(prep.q_bar, prep.k_bar, rho, nu)
    O = forward(prep, v, sel, heads=heads, qblocks=qblocks, quant=quant)
    return O, prep, sel
