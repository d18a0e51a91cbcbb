"""One SageSLA layer with its (batch, head) pairs split over ranks, one process per GPU.

"TurboDiffusion Demystified", section "Future Outlook and Community", names parallel
infrastructure as the next step. For this path it is plain data parallelism over heads:
every (b, h) pair is independent (its smoothing mean, scales, block lists, linear states
and output depend only on that head's Q, K and V), so a layer's B*H heads can be cut
into contiguous ranges, one per rank, and each rank runs prepare -> select -> forward on
its own range through the C ABI with no exchange at all. Only a consumer that needs the
whole output on every rank needs a collective: one all-gather of the per-rank outputs
(NCCL over NVLink/NVSwitch on GPUs; any torch.distributed backend works).

Layout: q, k, v, out are [B, H, N, d] contiguous, so the flattened heads [B*H, N, d] of
rank r are one contiguous slice [lo_r, hi_r) and the per-rank call sees shape
(B=1, H=hi_r-lo_r). The split is balanced: the first (B*H mod world) ranks take one extra
head. The all-gather pads every rank's block to the largest count so that all ranks send
equal sizes, then drops the padding.

No kernel here reads another GPU's memory: the only cross-GPU traffic is the library
collective on the gathered outputs.
"""
from __future__ import annotations

import torch

from . import sagesla as S


def head_range(n_heads: int, rank: int, world: int):
    """[lo, hi) of the flattened (b, h) heads owned by `rank` (balanced, contiguous)."""
    if not (0 <= rank < world) or n_heads < 1:
        raise ValueError("bad rank, world or head count")
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def local_heads(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """The rank's heads of a [B, H, N, d] tensor as a [1, h_r, N, d] view (no copy)."""
    B, H, N, d = x.shape
    lo, hi = head_range(B * H, rank, world)
    return x.reshape(B * H, N, d)[lo:hi].unsqueeze(0)


def gather_heads(out_local: torch.Tensor, B: int, H: int, group=None) -> torch.Tensor:
    """All-gather the ranks' [1, h_r, N, d] outputs into the full [B, H, N, d] output."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    _, h_r, N, d = out_local.shape
    width = -(-(B * H) // world)  # the largest per-rank head count
    send = out_local.new_zeros(width, N, d)
    send[:h_r] = out_local[0]
    if dist.get_backend(group) == "nccl":
        full = out_local.new_empty(world * width, N, d)
        dist.all_gather_into_tensor(full, send, group=group)
        parts = list(full.view(world, width, N, d))
    else:
        parts = [torch.empty_like(send) for _ in range(world)]
        dist.all_gather(parts, send, group=group)
    pieces = []
    for r in range(world):
        lo, hi = head_range(B * H, r, world)
        pieces.append(parts[r][: hi - lo])
    return torch.cat(pieces, 0).view(B, H, N, d)


class HeadParallelSageSLA:
    """SageSLA for one layer with its heads split over the ranks of a process group.

    Call with the rank's own heads (``local_heads`` of the full tensors, or the rank's
    share produced directly by its QKV projection); ``gather=True`` returns the full
    output on every rank, else the rank's [1, h_r, N, d] part.
    """

    def __init__(self, B, H, N, rho, nu, rank, world, device="cuda", group=None, engine=None):
        self.B, self.H, self.N = B, H, N
        self.rank, self.world, self.group = rank, world, group
        self.lo, self.hi = head_range(B * H, rank, world)
        self.engine = engine if engine is not None else S.SageSLA(
            1, self.hi - self.lo, N, rho, nu, device=device)

    def __call__(self, q_local, k_local, v_local, gather=True, stream=None):
        out = self.engine(q_local, k_local, v_local, stream=stream)
        if not gather or self.world == 1:
            return out
        return gather_heads(out, self.B, self.H, self.group)

    def check(self, stream=None):
        self.engine.check(stream)
