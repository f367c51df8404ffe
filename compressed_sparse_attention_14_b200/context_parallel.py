"""Context-parallel prefill of one long sequence across ranks.

[Walk §4.2 "long-context context parallelism"; Notes §2.5, "context
parallelism for long context"]: plain sequence sharding breaks compressed
attention in two places. A block of m tokens, and the overlapping b-window of
the next block, can straddle a rank boundary; and the ranks' compressed
lengths differ. The pages' two-stage exchange fixes both:

  1. rank i sends its last m uncompressed rows to rank i + 1, which
     compresses them together with its own rows (they are the b-window of
     its first block);
  2. an all-gather collects every rank's compressed entries, and a
     select-and-pad step rebuilds the complete compressed KV on every rank.

Each rank then runs the lightning indexer, top-k and sparse MQA for its own
queries against the complete caches (the causal rule only ever shows a query
entries that end before it, so every rank needs the entries of the ranks
before it, and none of the ones after).

Layout: rank r holds tokens [start_r, start_r + n_r) of the sequence, in rank
order, with start_0 = `start` and every n_r a multiple of m (blocks never
straddle ranks; the halo carries only the b-window). The m rows a rank sends
are hidden states: the receiver projects them with the same weights, which
gives the same projected rows as the sender's. Equal n_r gather straight into
the caches; unequal n_r are padded to the longest, gathered, and the valid
rows of each rank copied into place (the select-and-pad step).

The compute steps are the library's kernels (`csa_compress_from_hidden`,
then `csa_prefill` without weights: the gathered caches already hold the
rank's own entries, so it only attends); the exchange is torch.distributed
(NCCL over NVLink on GPUs). Every rank takes the same collective steps in the
same order, and every argument check that can fail runs on every rank before
the first data exchange, so a bad argument raises on all ranks together.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist


@dataclass
class PrefillOps:
    """The compute steps the exchange is wrapped around; by default the
    library's CUDA entry points.

    compress_from_hidden(x, W, bias, m, x_left) -> entries [n/m, c]
    prefill(x, x_left, W_kv, B_kv, W_idx, B_idx, start, kv_cache, idx_cache,
            qI, w, q, k, m, scale, sink) -> (out, lse)
    """
    compress_from_hidden: Callable
    prefill: Callable


def cuda_ops() -> PrefillOps:
    from . import csa_compress_from_hidden, csa_prefill

    def compress(x, W, bias, m, x_left):
        return csa_compress_from_hidden(x, W, bias, m, x_left=x_left)

    def prefill(x, x_left, W_kv, B_kv, W_idx, B_idx, start, kv_cache, idx_cache, qI, w, q, k, m, scale, sink):
        # the all-gather has put this rank's entries into the caches already:
        # no weights, so csa_prefill attends without compressing again
        return csa_prefill(x, None, None, None, None, None, start, kv_cache, idx_cache, qI, w, q, k, m=m,
                           scale=scale, sink=sink)

    return PrefillOps(compress_from_hidden=compress, prefill=prefill)


def chunk_layout(start: int, sizes: list[int], m: int) -> list[tuple[int, int]]:
    """(first token, first compressed entry) of every rank's chunk."""
    out, pos = [], start
    for n in sizes:
        out.append((pos, pos // m))
        pos += n
    return out


def _gather_shapes(vals: list[int], device, group) -> list[list[int]]:
    """Every rank's small integer vector (chunk size, whether it has left
    rows, cache capacities, start, m), so that all ranks run the same checks."""
    world = dist.get_world_size(group)
    mine = torch.tensor(vals, dtype=torch.int64, device=device)
    every = [torch.zeros_like(mine) for _ in range(world)]
    dist.all_gather(every, mine, group=group)
    return [[int(v) for v in t.tolist()] for t in every]


def _exchange_halo(x: torch.Tensor, x_left: Optional[torch.Tensor], m: int, group):
    """Stage 1: rank r's last m rows go to rank r + 1. Returns the rows this
    rank compresses its first block against (the caller's x_left on rank 0)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    send_req = None
    if rank + 1 < world:
        tail = x[x.shape[0] - m:].contiguous()
        send_req = dist.isend(tail, dist.get_global_rank(group, rank + 1) if group is not None else rank + 1,
                              group=group)
    left = x_left
    if rank > 0:
        left = torch.empty((m, x.shape[1]), dtype=x.dtype, device=x.device)
        dist.recv(left, dist.get_global_rank(group, rank - 1) if group is not None else rank - 1, group=group)
    if send_req is not None:
        send_req.wait()
    return left


def _gather_entries(local: torch.Tensor, cache: torch.Tensor, layout, sizes: list[int], m: int, group) -> None:
    """Stage 2: every rank's compressed entries into every rank's cache rows
    (select-and-pad when the ranks' entry counts differ)."""
    counts = [n // m for n in sizes]
    if len(set(counts)) == 1:
        views = [cache[e0:e0 + counts[0]] for (_, e0) in layout]
        dist.all_gather(views, local.contiguous(), group=group)
        return
    e_max = max(counts)
    pad = torch.zeros((e_max,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    bufs = [torch.empty_like(pad) for _ in counts]
    dist.all_gather(bufs, pad, group=group)
    for (_, e0), e, buf in zip(layout, counts, bufs):
        cache[e0:e0 + e] = buf[:e]


def csa_prefill_context_parallel(x, x_left, W_kv, B_kv, W_idx, B_idx, start: int, kv_cache, idx_cache, qI, w, q,
                                 k: int, m: int = 4, scale: float = 0.0, sink=None, group=None,
                                 ops: Optional[PrefillOps] = None):
    """This rank's part of a prefill chunk split over the ranks of `group`.

    x [n_r, d], qI [n_r, HI, cI], w [n_r, HI], q [n_r, H, c]: this rank's
    tokens (rank order along the sequence); x_left [m, d]: the m hidden rows
    before rank 0's first token (rank 0 only; None at the sequence start);
    start: rank 0's first token position (a multiple of m); kv_cache [Nmax, c]
    and idx_cache [Nmax, cI]: this rank's full copies, rows before start/m
    already filled. Returns (out [n_r, H, c], lse [n_r, H]) for this rank's
    queries; the caches end up holding the entries of every rank's tokens."""
    ops = ops or cuda_ops()
    rank = dist.get_rank(group)
    shapes = _gather_shapes([x.shape[0], int(x_left is not None), kv_cache.shape[0], idx_cache.shape[0], start, m],
                            x.device, group)
    sizes = [v[0] for v in shapes]
    if len({(v[4], v[5]) for v in shapes}) != 1 or m < 1 or start % m or any(n <= 0 or n % m for n in sizes):
        raise ValueError(f"every rank needs the same m and start (start a multiple of m) and a positive multiple "
                         f"of m tokens (chunk sizes {sizes}, (start, m) {[(v[4], v[5]) for v in shapes]})")
    total_entries = (start + sum(sizes)) // m
    room = min(min(v[2], v[3]) for v in shapes)
    if room < total_entries:
        raise ValueError(f"a rank's caches hold {room} entries, {total_entries} needed")
    if start > 0 and not shapes[0][1]:
        raise ValueError("rank 0 needs x_left when start > 0")
    layout = chunk_layout(start, sizes, m)
    my_start = layout[rank][0]

    left = _exchange_halo(x, x_left, m, group)
    if my_start == 0:
        left = None
    kv_local = ops.compress_from_hidden(x, W_kv, B_kv, m, left)
    idx_local = ops.compress_from_hidden(x, W_idx, B_idx, m, left)
    _gather_entries(kv_local, kv_cache, layout, sizes, m, group)
    _gather_entries(idx_local, idx_cache, layout, sizes, m, group)
    return ops.prefill(x, left, W_kv, B_kv, W_idx, B_idx, my_start, kv_cache, idx_cache, qI, w, q, k, m, scale,
                       sink)
