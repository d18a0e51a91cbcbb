"""The SFU exponential-rate probe (the denominator of the attention kernel's SFU floor).

Every CTA must report the exponentials it evaluated exactly (threads x chains x iterations,
two per instruction for the f16x2 and bf16x2 forms), a positive cycle count, and a per-SM
rate that is plausible and consistent across the SMs: the CTAs run the same loop, one per SM.
"""
import numpy as np
import pytest
import torch

from quantized_block_sparse_b200 import sagesla as S
from tests.gpu_helpers import ensure_lib

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", [0, 1, 2])
def test_ex2_probe_reports_consistent_rates(form):
    ensure_lib()
    n = torch.cuda.get_device_properties(0).multi_processor_count
    out = torch.full((3 * n,), -1, dtype=torch.int64, device="cuda")
    iters = 512
    S.sagesla_probe_ex2(form, iters, out)
    torch.cuda.synchronize()
    a = out.view(n, 3).cpu().numpy()
    per_instr = 2 if form in (1, 2) else 1
    assert (a[:, 0] == per_instr * 1024 * 8 * iters).all()
    assert (a[:, 1] > 0).all()
    assert ((a[:, 2] >= 0) & (a[:, 2] < 4 * n)).all()
    rate = a[:, 0] / a[:, 1]
    med = float(np.median(rate))
    # between 1 and 256 exponentials per SM clock, and no SM far off the median
    assert 1.0 <= med <= 256.0, med
    assert rate.min() > 0.5 * med and rate.max() < 1.5 * med, (rate.min(), med, rate.max())


def test_ex2_probe_rejects_a_short_buffer():
    ensure_lib()
    out = torch.zeros(8, dtype=torch.int64, device="cuda")
    L = S.lib()
    assert L.sagesla_probe_ex2(0, 64, 3, S._ptr(out), out.numel(), S._stream()) == 1
