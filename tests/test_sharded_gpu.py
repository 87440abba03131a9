"""The sequence-sharded forward and backward on one GPU: shards run one after
another in this process, no collective. The reassembled shards are checked
against the fp64 oracle on the whole batch (the forward's and the backward's
parity rules), and, since every (sequence, head) is computed independently of
the others, also for bit-exact agreement with one whole-batch call."""
import pytest
import torch

import oracle
from gated_delta_rule_114_b200 import sharded
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_bwd_grads, make_fwd_inputs
from parity_util import BF16_REL, BF16_STORE, check_bf16_out, check_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3])
def test_shards_equal_one_call(cuda_lib, world):
    w = WORKLOADS["ckda_varlen_N32_H32_d128"]
    lens = [300, 64, 1, 700, 129, 0, 250, 64]
    cu = torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32)
    inp = make_fwd_inputs(w, cu_seqlens=cu, H=4)
    d = to_dev(inp)
    o_all, sf_all = sharded._cuda_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                      d["initial_state"], inp["cu_seqlens"], 64, 1.0)
    o_parts, s_parts = [], []
    for r in range(world):
        o, sf, _ = sharded.fwd_chunked_sharded(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                               d["initial_state"], cu.tolist(), rank=r,
                                               world=world, chunk=64)
        o_parts.append(o)
        s_parts.append(sf)
    torch.cuda.synchronize()
    o_ref, sf_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               inp["initial_state"], inp["cu_seqlens"], 1.0)
    check_bf16_out(torch.cat(o_parts), o_ref, "o (shards)")
    check_close(torch.cat(s_parts), sf_ref, 1e-2, 0.0, "final_state (shards)")
    assert torch.equal(torch.cat(o_parts), o_all)
    assert torch.equal(torch.cat(s_parts), sf_all)


def test_bwd_shards_equal_one_call(cuda_lib):
    w = WORKLOADS["ckda_varlen_N32_H32_d128"]
    lens = [100, 0, 37, 200, 16, 64]
    cu = torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32)
    inp = make_fwd_inputs(w, cu_seqlens=cu, H=2)
    g = make_bwd_grads(w, int(cu[-1]), 2, len(lens))
    d = to_dev(inp)
    gd = to_dev(g)
    ref = sharded._cuda_bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["initial_state"],
                            gd["d_o"], gd["d_final_state"], inp["cu_seqlens"], 1.0)
    parts = [[] for _ in range(6)]
    for r in range(3):
        out = sharded.bwd_sharded(d["q"], d["k"], d["v"], d["alpha"], d["beta"], gd["d_o"],
                                  d["initial_state"], gd["d_final_state"], cu.tolist(),
                                  rank=r, world=3)
        for i in range(6):
            parts[i].append(out[i])
    torch.cuda.synchronize()
    want = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], g["d_o"],
                      inp["initial_state"], g["d_final_state"], inp["cu_seqlens"], 1.0)
    names = ["dq", "dk", "dv", "dalpha", "dbeta", "d_initial_state"]
    for i, name in enumerate(names):
        store = BF16_STORE if name in ("dq", "dk", "dv") else 0.0
        check_close(torch.cat(parts[i]), want[i], BF16_REL, store, name + " (shards)")
    for i in range(6):
        assert torch.equal(torch.cat(parts[i]), ref[i]), i
