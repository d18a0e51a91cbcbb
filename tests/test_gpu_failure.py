"""Failure detection on the GPU, without a fault.

Every kernel of the library waits on mbarriers through a bounded wait that, when its
limit runs out, sets the timeout bit of the caller's status word and lets the kernel
return. These tests make that path run on purpose: sagesla_selftest_wait_timeout launches
a kernel whose barrier nothing ever arrives on, with a short limit, so its wait must run
out. The status word must then read SAGESLA_ERR_TIMEOUT, the CUDA context must still work
(a normal SageSLA call afterwards is correct), and clearing the word must clear the status.
A second test writes the status word from the host and checks that sagesla_check_status
reports exactly what the word holds.
"""
import numpy as np
import pytest
import torch

import oracle as O
from quantized_block_sparse_b200 import sagesla as S
from quantized_block_sparse_b200.inputs import make_qkv
from tests.gpu_helpers import assert_output_close, ensure_lib, f32

pytestmark = pytest.mark.gpu

OK, CUDA_ERR, TIMEOUT = 0, 3, 4


def _status(ws):
    return S.lib().sagesla_check_status(S._ptr(ws), S._stream())


def test_bounded_wait_times_out_and_context_survives():
    ensure_lib()
    ws = S.alloc_workspace(1, 2, 1024)
    assert _status(ws) == OK
    import time
    t0 = time.perf_counter()
    S.sagesla_selftest_wait_timeout(ws, limit_us=20000)  # 20 ms
    assert _status(ws) == TIMEOUT
    assert time.perf_counter() - t0 < 5.0  # the wait ended by its own limit
    # the context is intact: clear the word and run a normal call on the same workspace
    S.lib().sagesla_reset_status(S._ptr(ws), ws.numel(), S._stream())
    assert _status(ws) == OK
    q, k, v = make_qkv(1, 2, (4, 16, 16), seed=0)
    eng = S.SageSLA(1, 2, 1024, 0.25, 0.25)
    out = eng(q.cuda(), k.cuda(), v.cuda())
    eng.check()
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, 0.25, 0.25)
    assert_output_close(out.float().cpu().numpy(), O.forward(prep, f32(v), sel))


def test_status_word_read_back_from_host():
    ensure_lib()
    ws = S.alloc_workspace(1, 1, 64)
    word = ws[:4].view(torch.int32)
    for value, expect in ((0, OK), (TIMEOUT, TIMEOUT), (TIMEOUT | 1, TIMEOUT), (1, CUDA_ERR)):
        word.fill_(value)
        assert _status(ws) == expect, value
    word.fill_(0)
    assert _status(ws) == OK


def test_selftest_rejects_bad_arguments():
    ensure_lib()
    L = S.lib()
    ws = S.alloc_workspace(1, 1, 64)
    assert L.sagesla_selftest_wait_timeout(S._ptr(ws), ws.numel(), 0, S._stream()) == 1
    assert L.sagesla_selftest_wait_timeout(S._ptr(ws), ws.numel(), 2000000, S._stream()) == 1
    assert L.sagesla_selftest_wait_timeout(S._ptr(ws), 64, 1000, S._stream()) == 1
    assert _status(ws) == OK  # nothing was launched
