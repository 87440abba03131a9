"""Sequence-sharded forward over several GPUs (one process per GPU).

Every (sequence, head) of the recurrence is independent, so a varlen batch
splits across ranks with no exchange on the data path: rank r takes a
contiguous range of whole sequences, chosen so that the ranks' token counts
are as even as contiguous ranges allow. The range's token rows are one
contiguous slice of the packed [T_total, H, d] inputs (no copy unless a slice
would start off a 16-byte boundary), its
cu_seqlens are the batch's entries rebased to 0, and the rank runs the same
C-ABI forward on its slice. Gathering the outputs is optional and is the only
collective (an all-gather of the per-rank o and final-state slices). The
backward pass shards the same way: a rank's gradients depend only on its own
sequences' rows (``bwd_sharded``).

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
    if int(cu_local[-1]) > 0:
        o_loc, sf_loc = fwd(qs, ks, vs, as_, bs, s0, cu_local, chunk, scale)
    else:  # no token rows (no sequences, or only empty ones): nothing to launch
        o_loc = torch.empty((0, H, d_v), dtype=q.dtype, device=q.device)
        sf_loc = (s0.clone() if s0 is not None else
                  torch.zeros((n1 - n0, H, d_k, d_v), dtype=torch.float32, device=q.device))
    if not gather:
        return o_loc, sf_loc, (n0, n1)
    return _gather(o_loc, sf_loc, cu_seqlens_host, world, group)


def _gather(o_loc, sf_loc, cu_seqlens_host, world, group):
    """All-gather the per-rank o and final-state slices and reassemble."""
    return _gather_parts([(o_loc, "rows"), (sf_loc, "seqs")], cu_seqlens_host, world, group)


def _gather_parts(parts, cu_seqlens_host, world, group):
    """All-gather per-rank slices, each indexed by token rows ("rows") or by
    sequences ("seqs"), padded to the largest rank's slice, and reassemble
    them in rank order."""
    cu = [int(x) for x in cu_seqlens_host]
    plan = plan_shards(cu, world)
    sizes = {"rows": [cu[n1] - cu[n0] for n0, n1 in plan], "seqs": [n1 - n0 for n0, n1 in plan]}

    def padded(x, m):
        out = torch.zeros((m,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        out[:x.shape[0]] = x
        return out

    out = []
    for x, kind in parts:
        n = sizes[kind]
        xs = [torch.empty_like(padded(x, max(n))) for _ in range(world)]
        dist.all_gather(xs, padded(x, max(n)), group=group)
        out.append(torch.cat([p[:c] for p, c in zip(xs, n)]))
    return tuple(out)


def _cuda_bwd(q, k, v, alpha, beta, s0, d_o, dsf, cu_local, scale, chunked=False):
    return ckda.bwd(q, k, v, alpha, beta, d_o, s0, dsf, cu_seqlens=cu_local.to(q.device),
                    cu_seqlens_host=cu_local, scale=scale, chunked=chunked)


def bwd_sharded(q, k, v, alpha, beta, d_o, initial_state, d_final_state, cu_seqlens_host,
                rank: int | None = None, world: int | None = None, *, scale: float = 1.0,
                gather: bool = False, group=None, bwd: Callable | None = None,
                chunked: bool = False):
    """This rank's shard of a packed varlen backward pass.

    Inputs are the whole batch (as for fwd_chunked_sharded, plus d_o
    [T_total, H, d_v] and d_final_state [N, H, d_k, d_v] or None); each rank
    reads only its own sequences' rows. Returns (dq, dk, dv, dalpha, dbeta,
    d_initial_state) for this rank's token rows and sequences and (n0, n1);
    with gather=True, the whole batch's gradients on every rank instead.
    `chunked` selects ckda_bwd_chunked for the shard; `bwd` replaces the CUDA
    backward (same arguments as the default) for host-side tests."""
    if rank is None:
        rank = dist.get_rank(group) if dist.is_initialized() else 0
    if world is None:
        world = dist.get_world_size(group) if dist.is_initialized() else 1
    if bwd is None:
        def bwd(*args):
            return _cuda_bwd(*args, chunked=chunked)
    n0, n1 = plan_shards(cu_seqlens_host, world)[rank]
    qs, ks, vs, as_, bs, s0, cu_local = shard_inputs(q, k, v, alpha, beta, initial_state,
                                                     cu_seqlens_host, n0, n1)
    cu = [int(x) for x in cu_seqlens_host]
    t0, t1 = cu[n0], cu[n1]

    def view(x):  # 16-byte aligned rows for the C ABI; copy a slice only if needed
        return x if x.data_ptr() % 16 == 0 else x.clone()

    dos = view(d_o[t0:t1])
    dsf = view(d_final_state[n0:n1]) if d_final_state is not None else None
    T, H, d_k = q.shape
    d_v = v.shape[2]
    if t1 > t0:
        grads = bwd(qs, ks, vs, as_, bs, s0, dos, dsf, cu_local, scale)
    else:  # no token rows: the initial-state gradient is the final-state one
        rows = lambda d, dt: torch.empty((0, H, d), dtype=dt, device=q.device)
        ds0 = (dsf.clone() if dsf is not None else
               torch.zeros((n1 - n0, H, d_k, d_v), dtype=torch.float32, device=q.device))
        grads = (rows(d_k, q.dtype), rows(d_k, q.dtype), rows(d_v, q.dtype),
                 rows(d_k, torch.float32), torch.empty((0, H), dtype=torch.float32, device=q.device),
                 ds0)
    if not gather:
        return tuple(grads) + ((n0, n1),)
    kinds = ["rows"] * 5 + ["seqs"]
    return _gather_parts(list(zip(grads, kinds)), cu_seqlens_host, world, group)
