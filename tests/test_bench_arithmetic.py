"""The bench's work counts against the hand-derived table of the measurement plan.

bench.py reports dense-equivalent TOPS (4*B*H*N^2*d per call) and the forward-level tensor
roofline from the executed work: 2*64*64*128 INT8 ops and as many BF16 flops per executed
(query block, critical key block) pair, plus 2*m*128*129 (marginal gather) and 2*64*128*129
(phi(Q~) H) BF16 flops per query block when m > 0. The figures below were derived by hand
from the workload shapes and the counts k_c = ceil(rho*nB), n_neg = floor(nu*nB), m = rest,
independently of this code; the test pins the bench's arithmetic to them.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle as O  # noqa: E402
from quantized_block_sparse_b200.inputs import WORKLOADS  # noqa: E402

# workload: (executed pairs, INT8 GOPs, BF16 GFLOPs, dense-equivalent TOPs per call)
TABLE = {
    # tiny: nB 16, k_c 4, m 8; BF16 = 128 pairs x 1048576 + 32 query blocks x
    # (2*8*128*129 + 2*64*128*129) = 134.2 M + 76.1 M
    "tiny": (128, 0.1342, 0.2103, 0.001074),
    "dense": (49152, 51.5, 51.5, 0.103),
    "480p": (319488, 335.0, 394.7, 6.594),
    "720p": (5626320, 5900.0, 6830.0, 117.05),
}


@pytest.mark.parametrize("name", sorted(TABLE))
def test_forward_work_matches_the_table(name):
    wl = WORKLOADS[name]
    nB = -(-wl.N // 64)
    k_c, n_neg, m = O.counts(nB, wl.rho, wl.nu)
    pairs, int8_g, bf16_g, dense_t = TABLE[name]
    assert wl.B * wl.H * nB * k_c == pairs
    w = bench.forward_work(wl, nB, k_c, m)
    assert w["int8_ops"] / 1e9 == pytest.approx(int8_g, rel=2e-3)
    assert w["bf16_flops"] / 1e9 == pytest.approx(bf16_g, rel=2e-3)
    assert bench.dense_equiv_ops(wl) / 1e12 == pytest.approx(dense_t, rel=5e-3)


def test_softmax_exponentials_at_480p():
    # one exponential per (query row, key) of every executed pair, plus one per element of
    # Q for phi(Q~): the figure the bench's SFU floor divides by the probed rate
    wl = WORKLOADS["480p"]
    nB = -(-wl.N // 64)
    k_c, _, m = O.counts(nB, wl.rho, wl.nu)
    pairs = wl.B * wl.H * nB * k_c
    exps = pairs * 64 * 64 + (wl.B * wl.H * wl.N * wl.d if m > 0 else 0)
    assert exps == 1_358_942_208
