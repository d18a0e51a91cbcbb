"""The no-allocation prepare entry point against the regular one.

sagesla_prepare_static_scratch serves callers that cannot allocate device memory when
they run prepare (an engine that owns all memory from start-up, a plugin host, a loop that
must not call cudaMalloc): its scratch is a fixed array inside the library. This test calls
it through the C ABI twice in a row, on two different inputs, and checks each result
against sagesla_prepare with a caller-provided workspace, bit for bit: both run the same
kernels on the same inputs, so every output (INT8 codes, scales, means, mu, h and z) must
be identical, and stale data left in the shared array by the previous call would show.
After each call the array's status word is read back and must be clean.

It lives in its own file, collected last, so a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

from quantized_block_sparse_b200 import sagesla as S
from quantized_block_sparse_b200.inputs import make_qkv, make_random_qkv
from tests.gpu_helpers import ensure_lib

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


def test_static_scratch_prepare_matches_workspace_prepare():
    ensure_lib()
    cases = [make_qkv(1, 2, (4, 16, 16), seed=0), make_random_qkv(2, 3, 1000, seed=5)]
    for q, k, v in cases:  # two calls in a row, different shapes and data
        B, H, N, _ = q.shape
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        ws = S.alloc_workspace(B, H, N)
        ref = S.sagesla_prepare(qd, kd, vd, ws)
        got = S.sagesla_prepare_static_scratch(qd, kd, vd)
        torch.cuda.synchronize()
        S.sagesla_check_status(ws)
        S.sagesla_static_scratch_status()
        for name in ("q8", "k8", "q_scale", "k_scale", "k_mean", "q_bar", "k_bar", "h", "z"):
            np.testing.assert_array_equal(_bits(getattr(got, name)), _bits(getattr(ref, name)),
                                          err_msg=name)


def test_static_scratch_rejects_oversized_shapes():
    ensure_lib()
    import ctypes
    sh = S._Shape(64, 64, 200000, 128)  # needs far more than the fixed scratch
    p = ctypes.c_void_p(0x1000)
    rc = S.lib().sagesla_prepare_static_scratch(ctypes.byref(sh), p, p, p, 0.088, *([p] * 9), None)
    assert rc == 2  # SAGESLA_ERR_UNSUPPORTED, nothing launched
