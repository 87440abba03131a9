"""Sequence-sharded forward over several GPUs (one process per GPU).

Every (sequence, head) of the recurrence is independent, so a varlen batch
splits across ranks with no exchange on the data path: rank r takes a
contiguous range of whole sequences, chosen so that the ranks' token counts
are as even as contiguous ranges allow. The range's token rows are one
contiguous slice of the packed [T_total, H, d] inputs (no copy unless a slice
would start off a 16-byte boundary), its
cu_seqlens are the batch's entries rebased to 0, and the rank runs the same
C-ABI forward on its slice. Gathering the outputs is optional and is the only
collective (an all-gather of the per-rank o and final-state slices).

The host logic (the split, the slicing, the reassembly) is plain Python and
runs under any torch.distributed backend; the forward itself is the CUDA
library's.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist

from gated_delta_rule_114_b200 import ckda


def plan_shards(cu_seqlens: Sequence[int], world: int) -> list[tuple[int, int]]:
    """Split sequences 0..N-1 into `world` contiguous ranges [n0, n1).

    Boundary r is placed at the sequence start closest to r/world of the
    tokens (never moving backwards), so every sequence is in exactly one range;
    ranges may be empty when there are fewer sequences than ranks."""
    cu = [int(x) for x in cu_seqlens]
    n_seq = len(cu) - 1
    if n_seq < 0 or world < 1:
        raise ValueError("need cu_seqlens with at least one entry and world >= 1")
    total = cu[-1] - cu[0]
    bounds = [0]
    for r in range(1, world):
        target = cu[0] + total * r / world
        n = bounds[-1]
        # advance while the next sequence start is at least as close to target
        while n < n_seq and abs(cu[n + 1] - target) <= abs(cu[n] - target):
            n += 1
        bounds.append(n)
    bounds.append(n_seq)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def shard_inputs(q, k, v, alpha, beta, initial_state, cu_seqlens_host: Sequence[int],
                 n0: int, n1: int):
    """Views of one shard: token rows cu[n0]..cu[n1] and sequences n0..n1."""
    cu = [int(x) for x in cu_seqlens_host]
    t0, t1 = cu[n0], cu[n1]
    cu_local = torch.tensor([c - t0 for c in cu[n0:n1 + 1]], dtype=torch.int32)

    def view(x):  # the C ABI takes 16-byte aligned rows; copy a slice only if it is not
        return x if x.data_ptr() % 16 == 0 else x.clone()

    s0 = view(initial_state[n0:n1]) if initial_state is not None else None
    return (view(q[t0:t1]), view(k[t0:t1]), view(v[t0:t1]), view(alpha[t0:t1]),
            view(beta[t0:t1]), s0, cu_local)


def _cuda_fwd(q, k, v, alpha, beta, s0, cu_local, chunk, scale):
    return ckda.fwd_chunked(q, k, v, alpha, beta, s0,
                            cu_seqlens=cu_local.to(q.device),
                            cu_seqlens_host=cu_local, chunk=chunk, scale=scale)


def fwd_chunked_sharded(q, k, v, alpha, beta, initial_state, cu_seqlens_host,
                        rank: int | None = None, world: int | None = None, *,
                        chunk: int = 0, scale: float = 1.0, gather: bool = False,
                        group=None, fwd: Callable | None = None):
    """This rank's shard of a packed varlen forward.

    Inputs are the whole batch (packed [T_total, H, d], cu_seqlens on the
    host); each rank reads only its own token rows. Returns (o_local,
    final_state_local, (n0, n1)); with gather=True, (o, final_state) of the
    whole batch on every rank instead. `fwd` replaces the CUDA forward (same
    arguments as the default) for host-side tests."""
    if rank is None:
        rank = dist.get_rank(group) if dist.is_initialized() else 0
    if world is None:
        world = dist.get_world_size(group) if dist.is_initialized() else 1
    fwd = fwd or _cuda_fwd
    n0, n1 = plan_shards(cu_seqlens_host, world)[rank]
    qs, ks, vs, as_, bs, s0, cu_local = shard_inputs(q, k, v, alpha, beta, initial_state,
                                                     cu_seqlens_host, n0, n1)
    T, H, d_k = q.shape
    d_v = v.shape[2]
    if n1 > n0:
        o_loc, sf_loc = fwd(qs, ks, vs, as_, bs, s0, cu_local, chunk, scale)
    else:
        o_loc = torch.empty((0, H, d_v), dtype=q.dtype, device=q.device)
        sf_loc = torch.empty((0, H, d_k, d_v), dtype=torch.float32, device=q.device)
    if not gather:
        return o_loc, sf_loc, (n0, n1)
    return _gather(o_loc, sf_loc, cu_seqlens_host, world, group)


def _gather(o_loc, sf_loc, cu_seqlens_host, world, group):
    """All-gather the per-rank slices (padded to the largest) and reassemble."""
    cu = [int(x) for x in cu_seqlens_host]
    plan = plan_shards(cu, world)
    rows = [cu[n1] - cu[n0] for n0, n1 in plan]
    seqs = [n1 - n0 for n0, n1 in plan]
    mr, ms = max(rows), max(seqs)

    def padded(x, m):
        out = torch.zeros((m,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        out[:x.shape[0]] = x
        return out

    o_parts = [torch.empty_like(padded(o_loc, mr)) for _ in range(world)]
    s_parts = [torch.empty_like(padded(sf_loc, ms)) for _ in range(world)]
    dist.all_gather(o_parts, padded(o_loc, mr), group=group)
    dist.all_gather(s_parts, padded(sf_loc, ms), group=group)
    o = torch.cat([p[:r] for p, r in zip(o_parts, rows)])
    sf = torch.cat([p[:s] for p, s in zip(s_parts, seqs)])
    return o, sf
