"""ctypes binding over libsagesla.so: argument marshalling only.

Every step of SageSLA runs in the CUDA library; this module allocates device tensors with
torch, passes their pointers and the current CUDA stream, and checks the status codes.
It raises if the library is missing: there is no CPU fallback.

Names follow the C ABI in include/sagesla.h: ``sagesla_counts``,
``sagesla_workspace_bytes``, ``sagesla_prepare``, ``sagesla_select``, ``sagesla_forward``,
``sagesla_check_status``.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

HEAD_DIM = 128
BLOCK = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsagesla.so")
_lib = None

_c_int_p = ctypes.POINTER(ctypes.c_int)
_vp = ctypes.c_void_p


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int)]


class SageSLAError(RuntimeError):
    pass


def lib():
    """Load libsagesla.so (built in-tree); fail loudly when it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise SageSLAError(
            f"{LIB_PATH} not found: build it with `python -m quantized_block_sparse_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sp = ctypes.POINTER(_Shape)
    L.sagesla_counts.argtypes = [sp, ctypes.c_double, ctypes.c_double, _c_int_p, _c_int_p, _c_int_p, _c_int_p]
    L.sagesla_counts.restype = ctypes.c_int
    L.sagesla_workspace_bytes.argtypes = [sp]
    L.sagesla_workspace_bytes.restype = ctypes.c_size_t
    L.sagesla_reset_status.argtypes = [_vp, ctypes.c_size_t, _vp]
    L.sagesla_reset_status.restype = ctypes.c_int
    L.sagesla_prepare.argtypes = [sp, _vp, _vp, _vp, ctypes.c_float] + [_vp] * 9 + [_vp, ctypes.c_size_t, _vp]
    L.sagesla_prepare.restype = ctypes.c_int
    L.sagesla_prepare_static_scratch.argtypes = [sp, _vp, _vp, _vp, ctypes.c_float] + [_vp] * 9 + [_vp]
    L.sagesla_prepare_static_scratch.restype = ctypes.c_int
    L.sagesla_static_scratch_status.argtypes = [_vp]
    L.sagesla_static_scratch_status.restype = ctypes.c_int
    L.sagesla_selftest_wait_timeout.argtypes = [_vp, ctypes.c_size_t, ctypes.c_uint, _vp]
    L.sagesla_selftest_wait_timeout.restype = ctypes.c_int
    L.sagesla_probe_ex2.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    L.sagesla_probe_ex2.restype = ctypes.c_int
    L.sagesla_backward_workspace_bytes.argtypes = [sp]
    L.sagesla_backward_workspace_bytes.restype = ctypes.c_size_t
    L.sagesla_backward.argtypes = ([sp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp,
                                    ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, _vp, _vp,
                                    ctypes.c_size_t, _vp])
    L.sagesla_backward.restype = ctypes.c_int
    L.sagesla_w8a8_quantize.argtypes = [_vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]
    L.sagesla_w8a8_quantize.restype = ctypes.c_int
    L.sagesla_w8a8_linear.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    L.sagesla_w8a8_linear.restype = ctypes.c_int
    L.sagesla_select.argtypes = [sp, _vp, _vp, ctypes.c_double, ctypes.c_double, _vp, _vp, _vp, _vp, _vp]
    L.sagesla_select.restype = ctypes.c_int
    L.sagesla_forward.argtypes = ([sp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int,
                                   _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp])
    L.sagesla_forward.restype = ctypes.c_int
    L.sagesla_marginal_sums.argtypes = [sp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.sagesla_marginal_sums.restype = ctypes.c_int
    L.sagesla_check_status.argtypes = [_vp, _vp]
    L.sagesla_check_status.restype = ctypes.c_int
    L.sagesla_status_string.argtypes = [ctypes.c_int]
    L.sagesla_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != 0:
        msg = lib().sagesla_status_string(rc).decode()
        raise SageSLAError(f"{what} failed: {msg} (status {rc})")


def _shape(B, H, N, d=HEAD_DIM):
    return _Shape(int(B), int(H), int(N), int(d))


def _require(ok: bool, what: str):
    """Argument check of the binding (kept under python -O)."""
    if not ok:
        raise SageSLAError(f"invalid argument: {what}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def softmax_scale(d: int = HEAD_DIM) -> float:
    """fl32(1/sqrt(d)) evaluated in double and rounded once to fp32 (host side)."""
    return float(np.float32(1.0 / math.sqrt(d)))


def sagesla_counts(B, H, N, rho, nu, d=HEAD_DIM):
    nB, kc, nn, m = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    sh = _shape(B, H, N, d)
    _check(lib().sagesla_counts(ctypes.byref(sh), float(rho), float(nu), ctypes.byref(nB),
                                ctypes.byref(kc), ctypes.byref(nn), ctypes.byref(m)), "sagesla_counts")
    return nB.value, kc.value, nn.value, m.value


def sagesla_workspace_bytes(B, H, N, d=HEAD_DIM) -> int:
    sh = _shape(B, H, N, d)
    n = lib().sagesla_workspace_bytes(ctypes.byref(sh))
    if n == 0:
        raise SageSLAError("invalid shape")
    return int(n)


def alloc_workspace(B, H, N, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(sagesla_workspace_bytes(B, H, N), dtype=torch.uint8, device=device)
    _check(lib().sagesla_reset_status(_ptr(ws), ws.numel(), _stream(stream)), "sagesla_reset_status")
    return ws


@dataclass
class Prepared:
    q8: torch.Tensor
    k8: torch.Tensor
    q_scale: torch.Tensor
    k_scale: torch.Tensor
    k_mean: torch.Tensor
    q_bar: torch.Tensor
    k_bar: torch.Tensor
    h: torch.Tensor
    z: torch.Tensor


@dataclass
class Selection:
    k_c: int
    n_neg: int
    m: int
    crit: torch.Tensor
    marg: torch.Tensor
    mask: torch.Tensor
    logits: torch.Tensor | None


def _dims(q):
    B, H, N, d = q.shape
    nB = -(-N // BLOCK)
    return B, H, N, d, nB


def alloc_prepared(B, H, N, device="cuda") -> Prepared:
    nB = -(-N // BLOCK)
    d = HEAD_DIM
    e = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=device)  # noqa: E731
    return Prepared(e(B, H, nB * BLOCK, d, dt=torch.int8), e(B, H, nB * BLOCK, d, dt=torch.int8),
                    e(B, H, nB), e(B, H, nB), e(B, H, d), e(B, H, nB, d), e(B, H, nB, d),
                    e(B, H, nB, d, d, dt=torch.bfloat16), e(B, H, nB, d))


def sagesla_prepare(q, k, v, workspace, sm_scale=None, out: Prepared | None = None, stream=None):
    """Steps 1-3 (+ block means and linear states). q, k, v: bf16 [B,H,N,128] on the GPU."""
    B, H, N, d, nB = _dims(q)
    for t in (q, k, v):
        _require(t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous() and t.shape == q.shape,
                 "inputs must be contiguous bf16 CUDA tensors of one shape")
    if out is None:
        out = alloc_prepared(B, H, N, q.device)
    c_s = softmax_scale(d) if sm_scale is None else float(sm_scale)
    sh = _shape(B, H, N, d)
    _check(lib().sagesla_prepare(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), c_s, _ptr(out.q8),
                                 _ptr(out.k8), _ptr(out.q_scale), _ptr(out.k_scale), _ptr(out.k_mean),
                                 _ptr(out.q_bar), _ptr(out.k_bar), _ptr(out.h), _ptr(out.z),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "sagesla_prepare")
    return out


def sagesla_prepare_static_scratch(q, k, v, sm_scale=None, out: Prepared | None = None, stream=None):
    """sagesla_prepare without a workspace: the library keeps the small scratch this step
    needs in its own fixed-size device array, for callers that cannot allocate here.
    Calls share that array, so order them on one stream."""
    B, H, N, d, nB = _dims(q)
    for t in (q, k, v):
        _require(t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous() and t.shape == q.shape,
                 "inputs must be contiguous bf16 CUDA tensors of one shape")
    if out is None:
        out = alloc_prepared(B, H, N, q.device)
    c_s = softmax_scale(d) if sm_scale is None else float(sm_scale)
    sh = _shape(B, H, N, d)
    _check(lib().sagesla_prepare_static_scratch(
        ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), c_s, _ptr(out.q8), _ptr(out.k8),
        _ptr(out.q_scale), _ptr(out.k_scale), _ptr(out.k_mean), _ptr(out.q_bar), _ptr(out.k_bar),
        _ptr(out.h), _ptr(out.z), _stream(stream)), "sagesla_prepare_static_scratch")
    return out


def sagesla_static_scratch_status(stream=None):
    """Raise if a bounded device wait of a static-scratch prepare gave up (synchronizes)."""
    _check(lib().sagesla_static_scratch_status(_stream(stream)), "static scratch status")


def alloc_selection(B, H, N, rho, nu, device="cuda", logits=False) -> Selection:
    nB, k_c, n_neg, m = sagesla_counts(B, H, N, rho, nu)
    nBp = -(-nB // 64) * 64
    crit = torch.empty(B, H, nB, k_c, dtype=torch.int32, device=device)
    marg = torch.empty(B, H, nB, max(m, 1), dtype=torch.int32, device=device)
    mask = torch.empty(B, H, nB, nBp, dtype=torch.bfloat16, device=device)
    lg = torch.empty(B, H, nB, nB, dtype=torch.float32, device=device) if logits else None
    return Selection(k_c, n_neg, m, crit, marg, mask, lg)


def sagesla_select(q_bar, k_bar, N, rho, nu, out: Selection | None = None, logits=False, stream=None):
    """Step 4. q_bar, k_bar: fp32 [B,H,nB,128]."""
    B, H, nB, d = q_bar.shape
    if out is None:
        out = alloc_selection(B, H, N, rho, nu, q_bar.device, logits)
    sh = _shape(B, H, N, d)
    _check(lib().sagesla_select(ctypes.byref(sh), _ptr(q_bar), _ptr(k_bar), float(rho), float(nu),
                                _ptr(out.crit), _ptr(out.marg) if out.m > 0 else None, _ptr(out.mask),
                                _ptr(out.logits), _stream(stream)), "sagesla_select")
    return out


def sagesla_forward(q, v, prep: Prepared, sel: Selection, workspace, out=None, sm_scale=None, stream=None):
    """Steps 5-7. Returns bf16 [B,H,N,128]."""
    B, H, N, d, nB = _dims(q)
    if out is None:
        out = torch.empty_like(q)
    c_s = softmax_scale(d) if sm_scale is None else float(sm_scale)
    sh = _shape(B, H, N, d)
    m = sel.m
    _check(lib().sagesla_forward(ctypes.byref(sh), _ptr(q), c_s, _ptr(prep.q8), _ptr(prep.k8),
                                 _ptr(prep.q_scale), _ptr(prep.k_scale), _ptr(v), _ptr(sel.crit), sel.k_c,
                                 _ptr(sel.mask), _ptr(sel.marg) if m > 0 else None, m, _ptr(prep.h),
                                 _ptr(prep.z), _ptr(out), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "sagesla_forward")
    return out


def sagesla_marginal_sums(mask, m, h, z, workspace, N=None, stream=None):
    """H_i = sum of h_j, Z_i = sum of z_j over the marginal blocks of each query block (the
    first half of step 6 on its own). mask bf16 [B,H,nB,nBp], h bf16 [B,H,nB,128,128],
    z fp32 [B,H,nB,128], N the token count (default 64 nB) -> (H bf16 like h, Z fp32 like z)."""
    B, H, nB = h.shape[:3]
    N = 64 * nB if N is None else int(N)
    _require(h.dtype == torch.bfloat16 and z.dtype == torch.float32 and mask.dtype == torch.bfloat16,
             "h bf16, z fp32 and mask bf16")
    Hout = torch.empty_like(h)
    Zout = torch.empty_like(z)
    _check(lib().sagesla_marginal_sums(ctypes.byref(_shape(B, H, N, HEAD_DIM)), _ptr(mask), int(m), _ptr(h),
                                       _ptr(z), _ptr(Hout), _ptr(Zout), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "sagesla_marginal_sums")
    return Hout, Zout


def sagesla_check_status(workspace, stream=None):
    _check(lib().sagesla_check_status(_ptr(workspace), _stream(stream)), "device status")


def sagesla_selftest_wait_timeout(workspace, limit_us: int, stream=None):
    """Diagnostics: run a kernel whose bounded wait must run out after limit_us (the
    failure path of every kernel); sagesla_check_status then reports the timeout."""
    _check(lib().sagesla_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(limit_us),
                                                _stream(stream)), "sagesla_selftest_wait_timeout")


def sagesla_probe_ex2(form: int, iters: int, out, stream=None):
    """Diagnostics: the SFU exponential-rate probe (form 0: ex2.approx.ftz.f32, 1: f16x2, 2: bf16x2)
    on out.numel() // 3 CTAs; out is an int64 CUDA tensor that receives, per CTA, the
    exponentials evaluated, the SM cycles taken and the SM id."""
    _require(out.dtype == torch.int64 and out.is_cuda and out.is_contiguous(),
             "out: contiguous int64 CUDA tensor")
    n = out.numel() // 3
    _check(lib().sagesla_probe_ex2(int(form), int(iters), n, _ptr(out), out.numel(), _stream(stream)),
           "sagesla_probe_ex2")


class SageSLA:
    """All three calls for one shape, with buffers allocated once (device memory via torch)."""

    def __init__(self, B, H, N, rho, nu, device="cuda", logits=False):
        self.B, self.H, self.N, self.rho, self.nu = B, H, N, rho, nu
        self.workspace = alloc_workspace(B, H, N, device)
        self.prep = alloc_prepared(B, H, N, device)
        self.sel = alloc_selection(B, H, N, rho, nu, device, logits)
        self.out = torch.empty(B, H, N, HEAD_DIM, dtype=torch.bfloat16, device=device)

    def __call__(self, q, k, v, stream=None, out=None):
        """One SageSLA call; the result goes to `out` (bf16 [B,H,N,128]) or the engine's own
        output buffer."""
        sagesla_prepare(q, k, v, self.workspace, out=self.prep, stream=stream)
        sagesla_select(self.prep.q_bar, self.prep.k_bar, self.N, self.rho, self.nu, out=self.sel,
                       stream=stream)
        return sagesla_forward(q, v, self.prep, self.sel, self.workspace,
                               out=self.out if out is None else out, stream=stream)

    def check(self, stream=None):
        sagesla_check_status(self.workspace, stream)


# ---------------------------------------------------------------- W8A8 linear layer
def sagesla_w8a8_quantize(x, stream=None):
    """bf16 [rows, K] -> (int8 codes [rows, K], fp32 scales [ceil(rows/128), ceil(K/128)])."""
    _require(x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous() and x.dim() == 2,
             "x: contiguous 2-D bf16 CUDA tensor")
    R, K = x.shape
    x8 = torch.empty(R, K, dtype=torch.int8, device=x.device)
    s = torch.empty(-(-R // 128), -(-K // 128), dtype=torch.float32, device=x.device)
    _check(lib().sagesla_w8a8_quantize(_ptr(x), R, K, _ptr(x8), _ptr(s), _stream(stream)),
           "sagesla_w8a8_quantize")
    return x8, s


def sagesla_w8a8_linear(x8, sx, w8, sw, bias=None, workspace=None, out=None, stream=None):
    """Y bf16 [M, N] = X W^T + bias from the quantized operands."""
    M, K = x8.shape
    N = w8.shape[0]
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=x8.device)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x8.device) if out is None else out
    _check(lib().sagesla_w8a8_linear(_ptr(x8), _ptr(sx), _ptr(w8), _ptr(sw), _ptr(bias), _ptr(y),
                                     M, N, K, _ptr(workspace), workspace.numel(), _stream(stream)),
           "sagesla_w8a8_linear")
    return y


# ---------------------------------------------------------------- backward
def sagesla_backward(q, k, v, dout, prep: Prepared, sel: Selection, sm_scale=None, workspace=None,
                     stream=None):
    """(dQ, dK, dV) fp32 [B,H,N,128] of the SageSLA output for upstream gradient dout (bf16),
    with the block lists of `sel` held fixed and the quantization read straight through."""
    B, H, N, d, nB = _dims(q)
    for t in (q, k, v, dout):
        _require(t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous() and t.shape == q.shape,
                 "inputs must be contiguous bf16 CUDA tensors of one shape")
    sh = _shape(B, H, N, d)
    if workspace is None:
        n = lib().sagesla_backward_workspace_bytes(ctypes.byref(sh))
        if n == 0:
            raise SageSLAError("invalid shape")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.empty(B, H, N, d, dtype=torch.float32, device=q.device) for _ in range(3))
    c_s = softmax_scale(d) if sm_scale is None else float(sm_scale)
    m = sel.m
    _check(lib().sagesla_backward(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), c_s,
                                  _ptr(prep.k_mean), _ptr(prep.h) if m > 0 else None,
                                  _ptr(prep.z) if m > 0 else None, _ptr(sel.crit), sel.k_c,
                                  _ptr(sel.mask) if m > 0 else None, m, _ptr(dq), _ptr(dk), _ptr(dv),
                                  _ptr(workspace), workspace.numel(), _stream(stream)),
           "sagesla_backward")
    return dq, dk, dv, workspace
