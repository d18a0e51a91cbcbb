"""C-ABI library checks that need no GPU: it loads, exports every declared symbol, and its
host-side logic (block counts, workspace size, argument validation) behaves.

Validation failures return before any CUDA call, so they run on a CPU-only machine.
"""
import ctypes
import os
import re

import pytest

import oracle as O
from quantized_block_sparse_b200 import sagesla as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sagesla.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(S.LIB_PATH):
        from quantized_block_sparse_b200.build import build
        build()
    return S.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sagesla_\w+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("sagesla_prepare", "sagesla_select", "sagesla_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


@pytest.mark.parametrize("N", [1, 63, 64, 65, 1000, 1024, 4096, 32760, 75600])
@pytest.mark.parametrize("rho,nu", [(0.25, 0.25), (1.0, 0.0), (0.1, 0.45), (0.2, 0.4),
                                    (0.05, 0.475), (0.5, 0.25), (0.3, 0.35), (0.15, 0.425)])
def test_counts_match_oracle(L, N, rho, nu):
    nB = -(-N // 64)
    got = S.sagesla_counts(1, 2, N, rho, nu)
    assert got == (nB,) + O.counts(nB, rho, nu)


def test_workspace_bytes(L):
    n = S.sagesla_workspace_bytes(1, 12, 32760)
    nB = 512
    assert n >= 12 * nB * 128 * 128 * 2  # H, bf16
    with pytest.raises(S.SageSLAError):
        S.sagesla_workspace_bytes(1, 12, 32760, d=64)


def _sh(B=1, H=2, N=1024, d=128):
    return S._Shape(B, H, N, d)


def test_validation_rejects_before_launch(L):
    sh = _sh()
    z = ctypes.c_int()
    # bad ratios
    assert L.sagesla_counts(ctypes.byref(sh), 0.0, 0.1, None, None, None, None) == 1
    assert L.sagesla_counts(ctypes.byref(sh), 0.5, 1.0, None, None, None, None) == 1
    assert L.sagesla_counts(ctypes.byref(sh), float("nan"), 0.1, None, None, None, None) == 1
    # unsupported head dim, empty shapes
    assert L.sagesla_counts(ctypes.byref(_sh(d=64)), 0.5, 0.1, ctypes.byref(z), None, None, None) == 2
    assert L.sagesla_counts(ctypes.byref(_sh(N=0)), 0.5, 0.1, None, None, None, None) == 1
    # limits: at most 8192 blocks of 64 tokens, at most 65535 (batch, head) pairs
    assert L.sagesla_counts(ctypes.byref(_sh(N=8192 * 64)), 0.5, 0.1, ctypes.byref(z), None, None, None) == 0
    assert L.sagesla_counts(ctypes.byref(_sh(N=8192 * 64 + 1)), 0.5, 0.1, None, None, None, None) == 2
    assert L.sagesla_counts(ctypes.byref(_sh(B=2, H=32768)), 0.5, 0.1, None, None, None, None) == 2
    assert L.sagesla_counts(None, 0.5, 0.1, None, None, None, None) == 1
    # null / misaligned device pointers are rejected without touching the GPU
    vp = [None] * 9
    assert L.sagesla_prepare(ctypes.byref(sh), None, None, None, 0.088, *vp, None, 0, None) == 1
    mis = ctypes.c_void_p(0x1001)
    args = [mis] * 3
    assert L.sagesla_prepare(ctypes.byref(sh), *args, 0.088, *([mis] * 9), mis, 1 << 30, None) == 1
    assert L.sagesla_select(ctypes.byref(sh), None, None, 0.25, 0.25, None, None, None, None, None) == 1
    assert L.sagesla_forward(ctypes.byref(sh), None, 0.088, None, None, None, None, None, None, 4,
                             None, None, 8, None, None, None, None, 0, None) == 1
    # k_c / m out of range
    p = ctypes.c_void_p(0x1000)
    assert L.sagesla_forward(ctypes.byref(sh), p, 0.088, p, p, p, p, p, p, 0,
                             p, p, 8, p, p, p, p, 1 << 40, None) == 1
    assert L.sagesla_forward(ctypes.byref(sh), p, 0.088, p, p, p, p, p, p, 4,
                             p, p, 13, p, p, p, p, 1 << 40, None) == 1
    # workspace too small
    assert L.sagesla_forward(ctypes.byref(sh), p, 0.088, p, p, p, p, p, p, 4,
                             p, p, 8, p, p, p, p, 16, None) == 1


def test_more_validation_paths(L):
    # every case below fails host-side checks, so no CUDA call is made
    sh = _sh()
    p = ctypes.c_void_p(0x1000)   # aligned, never dereferenced
    mis = ctypes.c_void_p(0x1008)  # 8-byte aligned only
    big = 1 << 40
    # prepare: softmax scale must be positive and finite; the workspace must be large enough
    for bad_scale in (0.0, -0.1, float("nan"), float("inf")):
        assert L.sagesla_prepare(ctypes.byref(sh), p, p, p, bad_scale, *([p] * 9), p, big, None) == 1
    assert L.sagesla_prepare(ctypes.byref(sh), p, p, p, 0.088, *([p] * 9), p, 64, None) == 1
    # select: ratios, the marginal list when m > 0, the optional logits buffer
    assert L.sagesla_select(ctypes.byref(sh), p, p, 1.5, 0.1, p, p, p, None, None) == 1
    assert L.sagesla_select(ctypes.byref(sh), p, p, 0.25, 0.25, p, None, p, None, None) == 1
    assert L.sagesla_select(ctypes.byref(sh), p, p, 0.25, 0.25, p, p, p, mis, None) == 1
    assert L.sagesla_select(ctypes.byref(sh), p, p, 0.25, 0.25, p, mis, p, None, None) == 1
    # the status word needs an aligned workspace of at least 256 bytes
    assert L.sagesla_reset_status(None, 1 << 20, None) == 1
    assert L.sagesla_reset_status(p, 128, None) == 1
    assert L.sagesla_reset_status(mis, 1 << 20, None) == 1
    # the no-workspace prepare: shape, pointers, scale, and the size of its fixed scratch
    args = [p] * 3 + [ctypes.c_float(0.088)] + [p] * 9 + [None]
    assert L.sagesla_prepare_static_scratch(None, *args) == 1
    assert L.sagesla_prepare_static_scratch(ctypes.byref(_sh(d=64)), *args) == 2
    assert L.sagesla_prepare_static_scratch(ctypes.byref(_sh(N=0)), *args) == 1
    assert L.sagesla_prepare_static_scratch(ctypes.byref(sh), *([mis] * 3), ctypes.c_float(0.088),
                                            *([p] * 9), None) == 1
    assert L.sagesla_prepare_static_scratch(ctypes.byref(sh), *([p] * 3), ctypes.c_float(float("nan")),
                                            *([p] * 9), None) == 1
    # 64 heads of 8192 blocks need 256 MiB of block sums: more than the fixed 24 MiB
    assert L.sagesla_prepare_static_scratch(ctypes.byref(_sh(H=64, N=8192 * 64)), *args) == 2
    # the failure-path self-test: workspace pointer and size, limit in 1..10^6 microseconds
    assert L.sagesla_selftest_wait_timeout(None, 1 << 20, 1000, None) == 1
    assert L.sagesla_selftest_wait_timeout(mis, 1 << 20, 1000, None) == 1
    assert L.sagesla_selftest_wait_timeout(p, 128, 1000, None) == 1
    assert L.sagesla_selftest_wait_timeout(p, 1 << 20, 0, None) == 1
    assert L.sagesla_selftest_wait_timeout(p, 1 << 20, 1000001, None) == 1
    # the SFU rate probe: form 0/1/2, iters in 1..2^20, 1..1024 CTAs, an aligned out of 3 per CTA
    assert L.sagesla_probe_ex2(3, 64, 4, p, 12, None) == 1
    assert L.sagesla_probe_ex2(-1, 64, 4, p, 12, None) == 1
    assert L.sagesla_probe_ex2(0, 0, 4, p, 12, None) == 1
    assert L.sagesla_probe_ex2(0, (1 << 20) + 1, 4, p, 12, None) == 1
    assert L.sagesla_probe_ex2(1, 64, 0, p, 12, None) == 1
    assert L.sagesla_probe_ex2(1, 64, 1025, p, 3 * 1025, None) == 1
    assert L.sagesla_probe_ex2(0, 64, 4, None, 12, None) == 1
    assert L.sagesla_probe_ex2(0, 64, 4, ctypes.c_void_p(0x1004), 12, None) == 1
    assert L.sagesla_probe_ex2(0, 64, 4, p, 11, None) == 1
    # the marginal sums on their own: m in 0..nB-1, aligned pointers, a large enough workspace
    # (shape N = 1024: nB = 16)
    assert L.sagesla_marginal_sums(ctypes.byref(sh), p, -1, p, p, p, p, p, big, None) == 1
    assert L.sagesla_marginal_sums(ctypes.byref(sh), p, 16, p, p, p, p, p, big, None) == 1
    assert L.sagesla_marginal_sums(ctypes.byref(sh), p, 4, p, mis, p, p, p, big, None) == 1
    assert L.sagesla_marginal_sums(ctypes.byref(sh), p, 4, p, p, None, p, p, big, None) == 1
    assert L.sagesla_marginal_sums(ctypes.byref(sh), p, 4, p, p, p, p, p, 256, None) == 1
    assert L.sagesla_marginal_sums(ctypes.byref(_sh(d=64)), p, 4, p, p, p, p, p, big, None) == 2


def test_status_strings(L):
    for code, word in [(0, b"ok"), (1, b"invalid"), (2, b"unsupported"), (3, b"CUDA"), (4, b"timed out")]:
        assert word in L.sagesla_status_string(code)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(S, "_lib", None)
    monkeypatch.setattr(S, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(S.SageSLAError):
        S.lib()


def test_binding_rejects_host_tensors_before_any_call():
    import torch
    q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)  # host memory: not a CUDA tensor
    with pytest.raises(S.SageSLAError, match="invalid argument"):
        S.sagesla_prepare(q, q, q, workspace=None)
    with pytest.raises(S.SageSLAError, match="invalid argument"):
        S.sagesla_w8a8_quantize(q[0, 0])
    with pytest.raises(S.SageSLAError, match="invalid argument"):
        S.sagesla_probe_ex2(0, 64, torch.zeros(3, dtype=torch.int64))
