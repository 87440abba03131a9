"""GPU parity of the complex-phase-gate forward against the oracle's
complex128 token recurrence (oracle.fwd_complex, pinned in
test_oracle_complex.py), for both entry points: ckda_fwd_complex (token-serial
kernel) and ckda_fwd_complex_chunked (16-token chunks, whose programs
test_complex_chunk_emu.py also runs on the CPU; its cases run after every
other GPU test). fp32 arithmetic: the fp32 check-mode bound,
max|x - x_ref| <= 1e-5 * rms(x_ref), on the real and imaginary parts of o and
of the final state."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_114_b200 import ckda
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_complex_inputs
from parity_util import FP32_REL, check_close, to_dev

pytestmark = pytest.mark.gpu


def custom(**kw):
    return dataclasses.replace(WORKLOADS["ckda_B1_H32_T8192_d128"], dtype="f32", **kw)


def lens_cu(lens):
    return torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))


IMPLS = pytest.mark.parametrize(
    "chunked", [False, pytest.param(True, marks=pytest.mark.last)], ids=["serial", "chunked"])


def parity(inp, scale, with_s0=True, use_cu=True, N=None, T=None, chunked=False):
    d = to_dev(inp)
    s0 = d["initial_state"] if with_s0 else None
    if use_cu:
        o, sf = ckda.fwd_complex(d["q"], d["k"], d["v"], d["alpha"], d["theta"], d["beta"], s0,
                                 cu_seqlens=d["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens"],
                                 scale=scale, chunked=chunked)
    else:
        o, sf = ckda.fwd_complex(d["q"], d["k"], d["v"], d["alpha"], d["theta"], d["beta"], s0,
                                 N=N, T=T, scale=scale, chunked=chunked)
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    o_ref, sf_ref = oracle.fwd_complex(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["theta"],
                                       inp["beta"], inp["initial_state"] if with_s0 else None,
                                       inp["cu_seqlens"], scale)
    for x, r, name in ((o, o_ref, "o"), (sf, sf_ref, "final_state")):
        xr = torch.view_as_real(x.cpu()).double().numpy()
        rr = np.stack([r.real, r.imag], axis=-1)
        check_close(xr, rr, FP32_REL, 0.0, name)
    return o, sf


@pytest.mark.parametrize("d_k,d_v,lens,ranges", [
    (16, 16, [5, 17, 0, 33], "sfda"),
    (64, 32, [64, 1, 40], "ckda"),
    (128, 128, [100, 37], "sfda"),
    (32, 64, [90], "ckda"),
])
@IMPLS
def test_complex_forward(cuda_lib, d_k, d_v, lens, ranges, chunked):
    w = custom(d_k=d_k, d_v=d_v, seed=900 + d_k + d_v)
    inp = make_complex_inputs(w, lens_cu(lens), H=2, ranges=ranges)
    parity(inp, 0.8, chunked=chunked)


@IMPLS
def test_complex_forward_without_initial_state(cuda_lib, chunked):
    w = custom(d_k=32, d_v=32, seed=931)
    parity(make_complex_inputs(w, lens_cu([20, 45]), H=2), 1.0, with_s0=False, chunked=chunked)


@IMPLS
def test_complex_forward_equal_lengths_without_cu_seqlens(cuda_lib, chunked):
    w = custom(d_k=64, d_v=64, seed=932)
    parity(make_complex_inputs(w, lens_cu([33, 33]), H=2), 1.0, use_cu=False, N=2, T=33,
           chunked=chunked)


@IMPLS
def test_complex_forward_is_deterministic(cuda_lib, chunked):
    w = custom(d_k=128, d_v=64, seed=933)
    d = to_dev(make_complex_inputs(w, lens_cu([70, 20]), H=2))
    a = ckda.fwd_complex(d["q"], d["k"], d["v"], d["alpha"], d["theta"], d["beta"],
                         d["initial_state"], cu_seqlens=d["cu_seqlens"], chunked=chunked)
    b = ckda.fwd_complex(d["q"], d["k"], d["v"], d["alpha"], d["theta"], d["beta"],
                         d["initial_state"], cu_seqlens=d["cu_seqlens"], chunked=chunked)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
