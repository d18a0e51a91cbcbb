"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: INT8 codes, scales, mu, block means, logits and block lists (near-ties are
counted, never expected here since the logits are bit-exact). Tolerance: the output,
cos >= 0.9995 and max error <= 2e-2 * max|O_ref| against the oracle's quantized path;
cos >= 0.99 against fp64 unquantized attention with the same blocks.
"""
import numpy as np
import pytest
import torch

import oracle as O
from quantized_block_sparse_b200.inputs import WORKLOADS, make_qkv, make_random_qkv, sweep_workload
from tests.gpu_helpers import (assert_linear_states_close, assert_output_close,
                               assert_prepare_bitexact, compare_lists, f32, run_gpu,
                               run_gpu_select)

pytestmark = pytest.mark.gpu


def _full_check(q, k, v, rho, nu, repeat=2):
    g = run_gpu(q, k, v, rho, nu, repeat=repeat)
    qf, kf, vf = f32(q), f32(k), f32(v)
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, rho, nu)
    assert_prepare_bitexact(g, prep)
    assert (g["k_c"], g["n_neg"], g["m"]) == (sel.k_c, sel.n_neg, sel.m)
    near = compare_lists(g, sel)
    assert near == 0
    B, H, N, _ = q.shape
    assert_linear_states_close(g, prep, vf, [(0, 0), (B - 1, H - 1)], N)
    ref = O.forward(prep, vf, sel)
    unq = O.forward(prep, vf, sel, quant=False)
    res = assert_output_close(g["out"], ref, unq)
    for o in g["outs"][1:]:  # deterministic run to run
        np.testing.assert_array_equal(o, g["outs"][0])
    return g, res


def test_tiny_workload():
    wl = WORKLOADS["tiny"]
    q, k, v = make_qkv(wl.B, wl.H, wl.grid, seed=0)
    _full_check(q, k, v, wl.rho, wl.nu)


def test_dense_workload_sageattention_only():
    wl = WORKLOADS["dense"]
    q, k, v = make_qkv(wl.B, wl.H, wl.grid, seed=0)
    g, res = _full_check(q, k, v, wl.rho, wl.nu)
    assert g["m"] == 0
    # against fp64 full softmax attention of the bf16 inputs
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), scale=float(O.softmax_scale(128))).numpy()
    from tests.gpu_helpers import cos
    assert cos(g["out"], ref) >= 0.99


@pytest.mark.parametrize("N,rho,nu", [
    (1, 1.0, 0.0),       # one token: a single block with 63 padded rows and keys
    (17, 0.5, 0.2),      # one ragged block smaller than a tile (nB = 1, so k_c = 1, m = 0)
    (40, 1.0, 0.0),
    (63, 0.3, 0.3),
    (130, 0.34, 0.33),   # three blocks, the last of 2 tokens: k_c = 2, n_neg = 0, m = 1
    (150, 0.25, 0.3),    # three blocks: k_c = 1, m = 2 (linear branch on a ragged tail)
    (64, 1.0, 0.0),      # a single block
    (65, 0.5, 0.0),      # two blocks, the second holds one token
    (100, 0.5, 0.5),     # ragged, no marginal blocks (m = 0), one negligible
    (191, 0.34, 0.33),   # odd number of blocks: the last CTA has one query block
    (1000, 0.25, 0.25),  # ragged tail, marginal branch on
    (2000, 0.1, 0.45),   # 480p-like ratios at a small size
    (4096, 1.0, 0.0),
])
def test_edge_shapes(N, rho, nu):
    q, k, v = make_random_qkv(1, 3, N, seed=N)
    _full_check(q, k, v, rho, nu)


def test_degenerate_blocks():
    # an all-zero Q block (s_q = 0), a K block equal to its channel mean (K~ = 0 -> s_k may
    # be tiny), identical key blocks (all logits tied) and a large outlier channel in K.
    q, k, v = make_random_qkv(1, 2, 640, seed=3)
    q[0, 0, 64:128] = 0
    k[0, 1] = k[0, 1, :64].repeat(10, 1)
    k[0, 0, :, 5] += 40.0
    _full_check(q, k, v, 0.3, 0.3)


def test_running_max_rises_every_tile():
    # Scores grow with the key block index (K_j = (j+1) * u + noise, Q aligned with u), so
    # the running row max rises by far more than 2^8 on every tile of the ascending walk and
    # the O rescale path runs on every tile; with rho < 1 also on union tiles of one half.
    g = torch.Generator().manual_seed(11)
    N = 1100
    u = torch.randn(128, generator=g, dtype=torch.float64)
    u = u / u.norm() * 9.0
    tok_blk = (torch.arange(N, dtype=torch.float64) // 64 + 1)[:, None]
    k = tok_blk * u[None, :] + 0.3 * torch.randn(N, 128, generator=g, dtype=torch.float64)
    q = u[None, :] + 0.3 * torch.randn(N, 128, generator=g, dtype=torch.float64)
    v = torch.randn(N, 128, generator=g, dtype=torch.float64)
    q, k, v = (x[None, None].repeat(1, 2, 1, 1).to(torch.bfloat16) for x in (q, k, v))
    _full_check(q, k, v, 1.0, 0.0)
    _full_check(q, k, v, 0.4, 0.2)


def test_batch_two_sweep_shape_small():
    wl = sweep_workload(0.2)
    q, k, v = make_qkv(2, 2, (3, 16, 32), seed=1)
    _full_check(q, k, v, wl.rho, wl.nu)


def _sampled_check(wl, heads_for_oracle, qblocks_per_head, seed=0):
    q, k, v = make_qkv(wl.B, wl.H, wl.grid, seed=seed)
    g = run_gpu(q, k, v, wl.rho, wl.nu, repeat=1)
    B, H, N, _ = q.shape
    nB = -(-N // 64)
    hs = slice(0, heads_for_oracle)
    qf, kf, vf = f32(q[:, hs]), f32(k[:, hs]), f32(v[:, hs])
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, wl.rho, wl.nu)
    assert_prepare_bitexact(g, prep, hs)
    near = compare_lists(g, sel, hs)
    rng = np.random.default_rng(7)
    qb = sorted(set(rng.choice(nB, size=qblocks_per_head, replace=False).tolist()) | {0, nB - 1})
    heads = [(b, h) for b in range(B) for h in range(heads_for_oracle)]
    ref = O.forward(prep, vf, sel, heads=heads, qblocks=qb)
    unq = O.forward(prep, vf, sel, heads=heads, qblocks=qb, quant=False)
    res = assert_output_close(g["out"][:, hs], ref, unq)
    return near, res


def test_480p_full_size_sampled():
    near, res = _sampled_check(WORKLOADS["480p"], heads_for_oracle=3, qblocks_per_head=24)
    assert near == 0


def test_720p_full_size_sampled():
    near, res = _sampled_check(WORKLOADS["720p"], heads_for_oracle=2, qblocks_per_head=12)
    assert near == 0


def test_480p_topk015_full_size_sampled():
    # --sla_topk 0.15: k_c = 77 critical blocks per row (odd), m = 205
    near, res = _sampled_check(WORKLOADS["480p_topk015"], heads_for_oracle=2, qblocks_per_head=12)
    assert near == 0


def test_480p_14b_full_size_sampled():
    # Wan2.1-14B at 480p: 40 heads; heads 0-1 compared against the oracle
    near, res = _sampled_check(WORKLOADS["480p_14b"], heads_for_oracle=2, qblocks_per_head=8)
    assert near == 0


def test_720p_i2v_full_size_sampled():
    near, res = _sampled_check(WORKLOADS["720p_i2v"], heads_for_oracle=1, qblocks_per_head=8, seed=1)
    assert near == 0


@pytest.mark.parametrize("rho", [1.0, 0.5, 0.2, 0.1, 0.05])
def test_sweep_full_size_sampled(rho):
    near, res = _sampled_check(sweep_workload(rho), heads_for_oracle=1, qblocks_per_head=8, seed=1)
    assert near == 0


@pytest.mark.parametrize("N", [90000, 140000, 270000])
def test_select_large_block_counts(N):
    # nB = 1407: row keys read from shared memory instead of registers; nB = 1407 and 2188:
    # 8 query-block rows per CTA, 4219: 4. Prepare and select only.
    q, k, v = make_random_qkv(1, 1, N, seed=N)
    g = run_gpu_select(q, k, v, 0.1, 0.45)
    prep = O.prepare(f32(q), f32(k))
    sel = O.select(prep.q_bar, prep.k_bar, 0.1, 0.45)
    assert_prepare_bitexact(g, prep)
    assert (g["k_c"], g["n_neg"], g["m"]) == (sel.k_c, sel.n_neg, sel.m)
    assert compare_lists(g, sel) == 0


def test_select_at_the_block_limit():
    # nB = 8192, the largest block count the library accepts (4 query-block rows per CTA).
    # Rows sampled for the exact check; every row checked for the list structure.
    N = 8192 * 64
    q, k, v = make_random_qkv(1, 1, N, seed=8)
    g = run_gpu_select(q, k, v, 0.1, 0.45)
    prep = O.prepare(f32(q), f32(k))
    assert_prepare_bitexact(g, prep)
    rows = np.sort(np.random.default_rng(0).choice(8192, 12, replace=False))
    sel = O.select(prep.q_bar[:, :, rows], prep.k_bar, 0.1, 0.45)
    assert (g["k_c"], g["n_neg"], g["m"]) == (sel.k_c, sel.n_neg, sel.m)
    np.testing.assert_array_equal(g["logits"][:, :, rows].view(np.uint32), sel.logits.view(np.uint32))
    np.testing.assert_array_equal(g["crit"][:, :, rows], sel.crit)
    np.testing.assert_array_equal(g["marg"][:, :, rows], sel.marg)
    crit, marg, mask = g["crit"][0, 0], g["marg"][0, 0], g["mask"][0, 0]
    assert (np.diff(crit, axis=1) > 0).all() and (np.diff(marg, axis=1) > 0).all()
    member = np.zeros((8192, 8192), dtype=np.int8)
    np.put_along_axis(member, crit.astype(np.int64), 1, axis=1)
    np.put_along_axis(member, marg.astype(np.int64), 2, axis=1)
    assert ((member == 1).sum(1) == sel.k_c).all() and ((member == 2).sum(1) == sel.m).all()
    np.testing.assert_array_equal(mask[:, :8192], (member == 2).astype(np.float32))


def test_whole_head_pairing_writes_every_row():
    # 800 blocks per head take the whole-head pairing of query blocks (a sequential greedy
    # over the head); a block missing from the tile list would leave its rows unwritten, so
    # the output starts as NaN and every real row must be finite afterwards. Sampled query
    # blocks of the first head are then checked against the oracle.
    import torch
    from quantized_block_sparse_b200 import sagesla as S
    from tests.gpu_helpers import ensure_lib
    ensure_lib()
    B, H, grid, rho, nu = 1, 2, (10, 40, 128), 0.1, 0.45  # N = 51200: nB = 800
    q, k, v = make_qkv(B, H, grid, seed=3)
    N = q.shape[2]
    eng = S.SageSLA(B, H, N, rho, nu)
    eng.out.fill_(float("nan"))
    out = eng(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    eng.check()
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    qf, kf, vf = f32(q[:, :1]), f32(k[:, :1]), f32(v[:, :1])
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, rho, nu)
    rng = np.random.default_rng(11)
    qb = sorted(set(rng.choice(800, size=10, replace=False).tolist()) | {0, 799})
    ref = O.forward(prep, vf, sel, heads=[(0, 0)], qblocks=qb)
    unq = O.forward(prep, vf, sel, heads=[(0, 0)], qblocks=qb, quant=False)
    assert_output_close(o[:, :1], ref, unq)
