"""The sequence-sharded forward and backward on one GPU: shards run one after
another in this process, no collective. Every (sequence, head) is computed independently
of the others, so the shards reassemble bit-exactly to one whole-batch call."""
import pytest
import torch

from gated_delta_rule_114_b200 import sharded
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_bwd_grads, make_fwd_inputs
from parity_util import to_dev

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
    for i in range(6):
        assert torch.equal(torch.cat(parts[i]), ref[i]), i
