"""Host logic of the head-sharded layer on CPU: the head partition, and the all-gather of
the per-rank outputs with two gloo ranks as spawned processes.

The CUDA path cannot run here, so each rank's engine is a stand-in: a per-head function of
the rank's own Q, K and V (no cross-head mixing, like SageSLA). The gathered output must
equal that function applied to the whole tensors, on every rank.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from quantized_block_sparse_b200.heads_parallel import head_range, local_heads  # noqa: E402


@pytest.mark.parametrize("n,world", [(12, 1), (12, 2), (12, 5), (40, 8), (3, 4), (1, 2), (7, 7)])
def test_head_range_partitions_and_balances(n, world):
    ranges = [head_range(n, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a, b), (c, _) in zip(ranges, ranges[1:]):
        assert b == c  # contiguous, disjoint, covering
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n
    assert sizes == sorted(sizes, reverse=True)  # the extra heads go to the first ranks


def test_head_range_rejects_bad_arguments():
    for args in [(12, -1, 2), (12, 2, 2), (0, 0, 1)]:
        with pytest.raises(ValueError):
            head_range(*args)


def test_local_heads_are_views_of_the_right_slice():
    x = torch.arange(2 * 3 * 5 * 4, dtype=torch.float32).view(2, 3, 5, 4)
    for r in range(4):
        lo, hi = head_range(6, r, 4)
        v = local_heads(x, r, 4)
        assert v.shape == (1, hi - lo, 5, 4)
        assert v.data_ptr() == x.view(6, 5, 4)[lo].data_ptr()
        assert torch.equal(v[0], x.view(6, 5, 4)[lo:hi])


def _per_head_fn(q, k, v):
    # stands in for the SageSLA engine: a per-head function of that head's inputs only
    return v * 2.0 + q.mean(dim=2, keepdim=True) - k.amax(dim=2, keepdim=True)


class _FakeEngine:
    def __call__(self, q, k, v, stream=None):
        return _per_head_fn(q, k, v)

    def check(self, stream=None):
        pass


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, B, H, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from quantized_block_sparse_b200.heads_parallel import HeadParallelSageSLA, local_heads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(B, H, 70, 8, generator=g) for _ in range(3))  # same on every rank
    layer = HeadParallelSageSLA(B, H, 70, 0.1, 0.45, rank, world, engine=_FakeEngine())
    full = layer(local_heads(q, rank, world), local_heads(k, rank, world),
                 local_heads(v, rank, world), gather=True)
    part = layer(local_heads(q, rank, world), local_heads(k, rank, world),
                 local_heads(v, rank, world), gather=False)
    ok_full = torch.equal(full, _per_head_fn(q, k, v))
    ok_part = torch.equal(part, _per_head_fn(*(local_heads(t, rank, world) for t in (q, k, v))))
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, ok_full, ok_part, tuple(full.shape)))


@pytest.mark.parametrize("B,H", [(1, 12), (2, 3)])  # 12 heads: 6 + 6; 6 heads: 3 + 3
def test_gathered_output_equals_the_whole_layer(B, H):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, B, H, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, ok_full, ok_part, shape) in enumerate(res):
        assert rank == r and ok_full and ok_part and shape == (B, H, 70, 8)


def test_ragged_split_gathers_with_padding():
    # 5 heads over 2 ranks: 3 + 2; the all-gather pads rank 1's block to 3 heads
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, 1, 5, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok_full and ok_part for _, ok_full, ok_part, _ in res)
