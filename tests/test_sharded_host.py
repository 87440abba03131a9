"""Host-side tests of the sequence-sharded forward and backward (no GPU): the
split, the slicing and the reassembly, with the fp64 oracle standing in for
the CUDA calls, in one process and across two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_114_b200 import sharded
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_bwd_grads, make_fwd_inputs

W = WORKLOADS["tiny_T64_d16_f32"]
LENS = [5, 40, 1, 0, 77, 33, 12, 64]


def cu_of(lens):
    return [0] + list(np.cumsum(lens))


def oracle_fwd(q, k, v, alpha, beta, s0, cu_local, chunk, scale):
    o, sf = oracle.fwd(q, k, v, alpha, beta, s0, cu_local, scale)
    return torch.from_numpy(np.asarray(o)), torch.from_numpy(np.asarray(sf))


@pytest.mark.parametrize("lens,world", [([10, 10, 10, 10], 2), ([100, 1, 1, 1], 2),
                                        (LENS, 3), ([7], 4), ([0, 0, 5], 2)])
def test_plan_shards_covers_every_sequence_once(lens, world):
    cu = cu_of(lens)
    plan = sharded.plan_shards(cu, world)
    assert len(plan) == world
    assert plan[0][0] == 0 and plan[-1][1] == len(lens)
    for (a0, a1), (b0, b1) in zip(plan, plan[1:]):
        assert a1 == b0 and a0 <= a1
    # balance: each boundary sits within one sequence of its token target
    total, longest = cu[-1], max(lens)
    for r, (n0, _) in enumerate(plan[1:], start=1):
        assert abs(cu[n0] - total * r / world) <= longest


def test_plan_shards_even_split():
    assert sharded.plan_shards(cu_of([10] * 8), 4) == [(0, 2), (2, 4), (4, 6), (6, 8)]


def inputs():
    inp = make_fwd_inputs(W, cu_seqlens=torch.tensor(cu_of(LENS), dtype=torch.int32), H=2)
    return inp


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_shards_reassemble_to_the_whole_batch(world):
    inp = inputs()
    cu = inp["cu_seqlens"].tolist()
    o_ref, sf_ref = oracle_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               inp["initial_state"], inp["cu_seqlens"], 0, 1.0)
    o_parts, s_parts = [], []
    for r in range(world):
        o, sf, (n0, n1) = sharded.fwd_chunked_sharded(
            inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["initial_state"],
            cu, rank=r, world=world, fwd=oracle_fwd)
        assert o.shape[0] == cu[n1] - cu[n0] and sf.shape[0] == n1 - n0
        o_parts.append(o)
        s_parts.append(sf)
    # each sequence's result depends only on its own rows: bit-identical
    assert torch.equal(torch.cat(o_parts), o_ref)
    assert torch.equal(torch.cat(s_parts), sf_ref)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = inputs()
        cu = inp["cu_seqlens"].tolist()
        o, sf = sharded.fwd_chunked_sharded(
            inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["initial_state"],
            cu, gather=True, fwd=oracle_fwd)
        if rank == 0:
            torch.save({"o": o, "sf": sf}, out)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_whole_batch(tmp_path):
    out = str(tmp_path / "gathered.pt")
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    got = torch.load(out)
    inp = inputs()
    o_ref, sf_ref = oracle_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               inp["initial_state"], inp["cu_seqlens"], 0, 1.0)
    assert torch.equal(got["o"], o_ref)
    assert torch.equal(got["sf"], sf_ref)


def oracle_bwd(q, k, v, alpha, beta, s0, d_o, dsf, cu_local, scale):
    r = oracle.bwd(q, k, v, alpha, beta, d_o, s0, dsf, cu_local, scale)
    return tuple(torch.from_numpy(np.asarray(x)) for x in r)


def bwd_case():
    inp = inputs()
    T, H = inp["q"].shape[:2]
    g = make_bwd_grads(W, T, H, len(LENS))
    return inp, g


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_bwd_shards_reassemble_to_the_whole_batch(world):
    inp, g = bwd_case()
    cu = inp["cu_seqlens"].tolist()
    ref = oracle_bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                     inp["initial_state"], g["d_o"], g["d_final_state"], inp["cu_seqlens"], 0.8)
    parts = [[] for _ in range(6)]
    for r in range(world):
        out = sharded.bwd_sharded(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                  g["d_o"], inp["initial_state"], g["d_final_state"], cu,
                                  rank=r, world=world, scale=0.8, bwd=oracle_bwd)
        n0, n1 = out[6]
        assert out[0].shape[0] == cu[n1] - cu[n0] and out[5].shape[0] == n1 - n0
        for i in range(6):
            parts[i].append(out[i].double())
    # every sequence's gradients depend only on its own rows: exact
    for i in range(6):
        assert torch.equal(torch.cat(parts[i]), ref[i].double()), i


def _bwd_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, g = bwd_case()
        res = sharded.bwd_sharded(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                  g["d_o"], inp["initial_state"], g["d_final_state"],
                                  inp["cu_seqlens"].tolist(), scale=0.8, gather=True,
                                  bwd=oracle_bwd)
        if rank == 0:
            torch.save(list(res), out)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_whole_backward(tmp_path):
    out = str(tmp_path / "gathered_bwd.pt")
    mp.spawn(_bwd_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    got = torch.load(out)
    inp, g = bwd_case()
    ref = oracle_bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                     inp["initial_state"], g["d_o"], g["d_final_state"], inp["cu_seqlens"], 0.8)
    for x, r in zip(got, ref):
        assert torch.equal(x.double(), r.double())
