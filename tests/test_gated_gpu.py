"""GPU parity of the fused input prologue (ckda_fwd_chunked_gated,
ckda_decode_step_gated) against the oracle's gate_prologue followed by its
token recurrence: tensor-core path (bf16), CUDA-core path (fp32 check mode
and bf16), decode; CKDA and KDA gate ranges."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_114_b200 import ckda
from gated_delta_rule_114_b200.inputs import (WORKLOADS, make_decode_state,
                                              make_gated_decode_tokens,
                                              make_gated_fwd_inputs)
from parity_util import (check_bf16_out, check_close, check_fp32, poison, select_seqs,
                         to_dev)

pytestmark = pytest.mark.gpu

GATES = {"ckda": dict(ckda.CKDA_GATES, k_eps=1e-6), "kda": dict(ckda.KDA_GATES, k_eps=1e-3)}


def custom(base, **kw):
    return dataclasses.replace(WORKLOADS[base], **kw)


def lens_cu(lens):
    return torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))


def run_gated(inp, gates, chunk, scale):
    d = to_dev(inp)
    o, sf = ckda.fwd_chunked_gated(d["q"], d["k_raw"], d["v"], d["a_logit"], d["c_logit"],
                                   ckda.GateParams(**gates), d["initial_state"],
                                   cu_seqlens=d["cu_seqlens"],
                                   cu_seqlens_host=inp["cu_seqlens"], chunk=chunk,
                                   scale=scale)
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    return o, sf


def ref_gated(inp, gates, scale):
    return oracle.fwd_gated(inp["q"], inp["k_raw"], inp["v"], inp["a_logit"],
                            inp["c_logit"], gates, inp["initial_state"],
                            inp["cu_seqlens"], scale)


@pytest.mark.parametrize("gname", ["ckda", "kda"])
@pytest.mark.parametrize("d_v", [128, 64])
def test_gated_tensor_core_bf16(cuda_lib, gname, d_v):
    w = custom("ckda_B1_H32_T8192_d128", d_v=d_v, seed=8100 + d_v)
    inp = make_gated_fwd_inputs(w, cu_seqlens=lens_cu([300, 64, 1, 130, 0, 77]), H=4)
    o, sf = run_gated(inp, GATES[gname], 64, 0.9)
    o_ref, sf_ref = ref_gated(inp, GATES[gname], 0.9)
    check_bf16_out(o, o_ref)
    check_close(sf, sf_ref, 1e-2, 0.0, "final_state")


def test_gated_partial_chunk_ignores_the_next_sequence(cuda_lib):
    """As in the plain forward: with the sequence after a partial chunk full
    of NaN and inf (q, raw k, v and both gate logits), the sequences around
    it match the oracle run on them alone."""
    keys = ("q", "k_raw", "v", "a_logit", "c_logit")
    w = custom("ckda_B1_H32_T8192_d128", seed=8300)
    inp = make_gated_fwd_inputs(w, cu_seqlens=lens_cu([100, 70, 29]), H=4)
    poison(inp, 100, 170, keys)
    o, sf = run_gated(inp, GATES["ckda"], 64, 1.0)
    sub, idx = select_seqs(inp, [0, 2], keys)
    o_ref, sf_ref = ref_gated(sub, GATES["ckda"], 1.0)
    check_bf16_out(o[idx], o_ref)
    check_close(sf[[0, 2]], sf_ref, 1e-2, 0.0, "final_state")


def test_gated_tensor_core_bf16_long(cuda_lib):
    """One 2048-token sequence, H=8: every chunk slot of the persistent prep."""
    w = custom("ckda_B1_H32_T8192_d128", seed=8200)
    inp = make_gated_fwd_inputs(w, cu_seqlens=lens_cu([2048]), H=8)
    o, sf = run_gated(inp, GATES["ckda"], 64, 1.0)
    o_ref, sf_ref = ref_gated(inp, GATES["ckda"], 1.0)
    check_bf16_out(o, o_ref)
    check_close(sf, sf_ref, 1e-2, 0.0, "final_state")


@pytest.mark.parametrize("d_k,d_v,chunk", [(64, 64, 32), (16, 16, 16), (128, 32, 64)])
def test_gated_cuda_core_fp32(cuda_lib, d_k, d_v, chunk):
    w = custom("ckda_B1_H32_T8192_d128", d_k=d_k, d_v=d_v, dtype="f32", seed=8300 + d_k)
    inp = make_gated_fwd_inputs(w, cu_seqlens=lens_cu([150, 1, 0, 70]), H=3)
    o, sf = run_gated(inp, GATES["ckda"], chunk, 1.25)
    o_ref, sf_ref = ref_gated(inp, GATES["ckda"], 1.25)
    check_fp32(o, o_ref, "o")
    check_fp32(sf, sf_ref, "final_state")


def test_gated_cuda_core_bf16(cuda_lib):
    w = custom("ckda_B1_H32_T8192_d128", d_k=64, d_v=128, seed=8400)
    inp = make_gated_fwd_inputs(w, cu_seqlens=lens_cu([100, 33]), H=2)
    o, sf = run_gated(inp, GATES["kda"], 32, 1.0)
    o_ref, sf_ref = ref_gated(inp, GATES["kda"], 1.0)
    check_bf16_out(o, o_ref)
    check_close(sf, sf_ref, 1e-2, 0.0, "final_state")


@pytest.mark.parametrize("dtype,d_k,d_v", [("bf16", 128, 128), ("f32", 64, 32)])
def test_gated_decode(cuda_lib, dtype, d_k, d_v):
    w = custom("decode_N256_H32_d128", d_k=d_k, d_v=d_v, dtype=dtype, seed=8500 + d_k)
    N, H = 8, 4
    state = make_decode_state(w, N=N, H=H)
    st_dev = state.cuda().contiguous()
    st_ref = state.double().numpy().copy()
    gates = GATES["ckda"]
    for step in range(4):
        tok = make_gated_decode_tokens(w, step, N=N, H=H)
        d = to_dev(tok)
        o = torch.empty((N, H, d_v), dtype=d["q"].dtype, device="cuda")
        ckda.ckda_decode_step_gated(d["q"], d["k_raw"], d["v"], d["a_logit"], d["c_logit"],
                                    st_dev, o, ckda.GateParams(**gates), scale=0.5)
        o_ref = oracle.decode_gated(tok["q"], tok["k_raw"], tok["v"], tok["a_logit"],
                                    tok["c_logit"], st_ref, gates, scale=0.5)
        torch.cuda.synchronize()
        if dtype == "f32":
            check_fp32(o, o_ref, "o step %d" % step)
        else:
            check_bf16_out(o, o_ref)
    if dtype == "f32":
        check_fp32(st_dev, st_ref, "state")
    else:
        check_close(st_dev, st_ref, 1e-2, 0.0, "state")
