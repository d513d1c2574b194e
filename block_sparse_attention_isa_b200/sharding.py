"""Head-parallel ISA forward over several GPUs (one process per GPU).

Every (batch, head) slice of the pass is independent through all five stages:
the pooling probe, the top-k, the sharpness and the routing are taken per
slice (papernotes.org notes, Key designs 1 and 3: the coarse map and the
sharpness are per batch and head). So the B*H slices are split into contiguous
ranges, one per rank, and each rank runs the single-GPU pass on its own range
with no collective on the data path. The only exchange is optional: when one
GPU must hold the whole output, the ranks all-gather O over NCCL (NVLink /
NVSwitch), each into its own buffer. No rank ever hands another GPU's memory to
a kernel or a copy engine of its own.

A rank's range of slices is a contiguous run of the [B, H, N, D] layout, so the
per-rank call is the ordinary C-ABI call on a [1, S_r, N, D] view: pointer
offsets only, no copy.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

__all__ = ["slice_range", "slice_counts", "forward_shard", "gather_output", "forward_sharded"]


def slice_counts(n_slices: int, world: int):
    """Slices per rank: the first n_slices % world ranks take one more."""
    if world <= 0 or n_slices < 0:
        raise ValueError("world must be positive and n_slices non-negative")
    base, extra = divmod(n_slices, world)
    return [base + (1 if r < extra else 0) for r in range(world)]


def slice_range(rank: int, world: int, n_slices: int) -> Tuple[int, int]:
    """[start, stop) of the flattened (batch, head) slices that `rank` computes."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    counts = slice_counts(n_slices, world)
    start = sum(counts[:rank])
    return start, start + counts[rank]


def _library_forward(q, k, v, out, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns):
    from block_sparse_attention_isa_b200 import forward_into
    forward_into(q, k, v, out, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns=alpha_ns)


def forward_shard(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float, rank: int, world: int,
                  out=None, alpha_ns: float = 0.0, compute: Optional[Callable] = None):
    """Run the pass on this rank's slice range of full [B, H, N, D] inputs.

    Returns (out_local [S_r, N, D], (start, stop)). `compute(q, k, v, out, L_src, L_ctx, b,
    alpha_s, alpha_f, alpha_ns)` computes one [1, S, N, D] batch into `out`; the default is the
    CUDA library.
    """
    B, H, N, D = q.shape
    start, stop = slice_range(rank, world, B * H)
    fn = compute or _library_forward
    qs, ks, vs = (t.reshape(B * H, N, D)[start:stop] for t in (q, k, v))
    if out is None:
        out = qs.new_empty(qs.shape)
    if stop > start:
        fn(qs.unsqueeze(0), ks.unsqueeze(0), vs.unsqueeze(0), out.unsqueeze(0), L_src, L_ctx, b, alpha_s, alpha_f,
           alpha_ns)
    return out, (start, stop)


def gather_output(out_local, B: int, H: int, group=None):
    """All-gather every rank's [S_r, N, D] output into a full [B, H, N, D] tensor on every rank.

    Ranks with fewer slices pad their chunk to the largest count, so that one fixed-size
    all-gather suffices; the padding is dropped afterwards.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    counts = slice_counts(B * H, world)
    S_max = max(counts)
    N, D = out_local.shape[1], out_local.shape[2]
    send = out_local
    if out_local.shape[0] < S_max:
        send = out_local.new_zeros((S_max, N, D))
        send[:out_local.shape[0]].copy_(out_local)
    recv = out_local.new_empty((world * S_max, N, D))
    dist.all_gather_into_tensor(recv, send.contiguous(), group=group)
    parts = [recv[r * S_max:r * S_max + counts[r]] for r in range(world)]
    return torch.cat(parts, dim=0).reshape(B, H, N, D)


def forward_sharded(q, k, v, L_src: int, L_ctx: int, b: int, alpha_s: float, alpha_f: float, group=None,
                    gather: bool = True, alpha_ns: float = 0.0, compute: Optional[Callable] = None):
    """The whole pass split over the ranks of `group` by (batch, head) slice.

    Each rank computes its contiguous range of slices; with `gather` the full output is
    all-gathered to every rank (returns [B, H, N, D]), otherwise the rank's own
    [S_r, N, D] part and its range are returned.
    """
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    out_local, rng = forward_shard(q, k, v, L_src, L_ctx, b, alpha_s, alpha_f, rank, world, alpha_ns=alpha_ns,
                                   compute=compute)
    if not gather:
        return out_local, rng
    B, H = q.shape[:2]
    return gather_output(out_local, B, H, group)
