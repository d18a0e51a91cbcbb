"""CPU oracle for the SageSLA backward pass (gradients of the attention output).  TEST
INFRASTRUCTURE ONLY: only the tests may import this module.

The pages call the sparse-linear attention "trainable" ("TurboDiffusion Demystified",
section "Pillar Two: Sparse-Linear Attention - SLA") and say nothing more about its
gradient. The reading taken here is the plainest one: the gradient of the forward
definition with the block selection held fixed (the lists are discrete, so they carry no
gradient) and the INT8 quantization read as the identity (the straight-through reading,
so the scores are Q~.K~ in full precision and P is not rounded). What stays
differentiable:

* the fold Q~ = c_s Q (c_s a constant);
* the smoothing K~ = K - mean_t K, a function of all of K;
* the softmax branch over each query block's critical key tokens;
* the linear branch phi(Q~) phi(K~)^T V / (phi(Q~) phi(K~)^T 1) over its marginal key
  tokens (zero where a row has none), with phi(x) = elu(x) + 1.

The forward is written densely over the real tokens with token-level masks built from
the block lists, in fp64 with torch, and autograd gives dQ, dK and dV for an upstream
gradient dO. The forward agrees with the pinned numpy oracle's unquantized path
(``sagesla_oracle.forward(..., quant=False)`` on an exact ``prepare``). The gradients are
pinned against central finite differences and against the shift invariance of the
method: adding a per-channel constant to K changes nothing, so dK sums to zero over tokens.
"""
from __future__ import annotations

import numpy as np
import torch

from .sagesla_oracle import BLOCK, Selection, softmax_scale


def _phi(x: torch.Tensor) -> torch.Tensor:
    return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))


def _token_mask(rows: np.ndarray, nB: int, N: int, b: int) -> torch.Tensor:
    """[N, N] bool: token t may use token u when u's block is in the list of t's block."""
    blk = torch.zeros(nB, nB, dtype=torch.bool)
    for i in range(nB):
        if rows.shape[1]:
            blk[i, torch.as_tensor(rows[i], dtype=torch.long)] = True
    tb = torch.arange(N) // b
    return blk[tb][:, tb]


def head_forward(q, k, v, crit_rows, marg_rows, c_s: float, b: int = BLOCK) -> torch.Tensor:
    """Output of one (batch, head): q, k, v torch fp64 [N, d]; lists [nB, k_c] / [nB, m]."""
    N = q.shape[0]
    nB = -(-N // b)
    qt = q * c_s
    kt = k - k.mean(dim=0, keepdim=True)
    crit = _token_mask(crit_rows, nB, N, b)
    s = (qt @ kt.T).masked_fill(~crit, float("-inf"))
    o = torch.softmax(s, dim=1) @ v
    if marg_rows.shape[1]:
        a = (_phi(qt) @ _phi(kt).T) * _token_mask(marg_rows, nB, N, b)
        den = a.sum(dim=1, keepdim=True)
        o = o + (a @ v) / torch.where(den > 0, den, torch.ones_like(den))
    return o


def forward_backward(q, k, v, do, sel: Selection, c_s=None, b: int = BLOCK):
    """O and (dQ, dK, dV) for upstream gradient dO; all [B,H,N,d] fp64 numpy arrays.

    q, k, v, do: float arrays [B,H,N,d]; sel: the block lists (its crit and marg are used).
    """
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, H, N, d = q.shape
    cs = float(softmax_scale(d) if c_s is None else c_s)
    O = np.empty_like(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    for bb in range(B):
        for hh in range(H):
            qh, kh, vh = (torch.tensor(x[bb, hh], requires_grad=True) for x in (q, k, v))
            o = head_forward(qh, kh, vh, sel.crit[bb, hh], sel.marg[bb, hh], cs, b)
            g = torch.autograd.grad(o, (qh, kh, vh), grad_outputs=torch.tensor(do[bb, hh]))
            O[bb, hh] = o.detach().numpy()
            dq[bb, hh], dk[bb, hh], dv[bb, hh] = (t.numpy() for t in g)
    return O, (dq, dk, dv)
