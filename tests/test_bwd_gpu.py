"""GPU parity of the backward pass against the oracle's fp64 adjoint
(oracle.bwd, pinned by finite differences in test_oracle_bwd.py), for both
entry points: ckda_bwd (token-serial kernel) and ckda_bwd_chunked (the
chunkwise kernel, whose per-CTA program test_bwd_chunk_emu.py also runs on
the CPU).

Tolerances follow the forward's rule (parity_util): fp32 I/O check mode
max|x - x_ref| <= BWD_FP32_REL * rms(x_ref) for every gradient; bf16 I/O
1e-2 * rms plus the bf16 store allowance 2^-8 |x_ref| for dq, dk, dv (stored
in bf16) and 1e-2 * rms for dalpha, dbeta and the initial-state gradient
(fp32). BWD_FP32_REL is ten times the forward's fp32 bound: the backward
runs the recurrence twice (the forward recompute and the adjoint), and dk,
dbeta are differences of two products (G w - S' g, g . w), which loses up to
a decade of relative precision against the rms of the result.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_114_b200 import ckda
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_bwd_grads, make_fwd_inputs
from parity_util import BF16_REL, BF16_STORE, check_close, to_dev

pytestmark = pytest.mark.gpu

BWD_FP32_REL = 1e-4
NAMES = ["dq", "dk", "dv", "dalpha", "dbeta", "d_initial_state"]


def custom(base, **kw):
    return dataclasses.replace(WORKLOADS[base], **kw)


def lens_cu(lens):
    return torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))


def case(w, lens, H, with_final=True, with_s0=True):
    cu = lens_cu(lens)
    inp = make_fwd_inputs(w, cu_seqlens=cu, H=H)
    if not with_s0:
        inp["initial_state"] = None
    elif inp["initial_state"] is None:
        g = torch.Generator().manual_seed(w.seed + 99)
        inp["initial_state"] = 0.1 * torch.randn(len(lens), H, w.d_k, w.d_v, generator=g)
    grads = make_bwd_grads(w, int(cu[-1]), H, len(lens))
    if not with_final:
        grads["d_final_state"] = None
    return inp, grads


# the chunkwise kernel's cases run after every other GPU test
IMPLS = pytest.mark.parametrize(
    "chunked", [False, pytest.param(True, marks=pytest.mark.last)], ids=["serial", "chunked"])


def run_gpu(inp, grads, scale, chunked=False):
    d = to_dev(inp)
    g = to_dev(grads)
    out = ckda.bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], g["d_o"], d["initial_state"],
                   g["d_final_state"], cu_seqlens=d["cu_seqlens"],
                   cu_seqlens_host=inp["cu_seqlens"], scale=scale, chunked=chunked)
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    return out


def run_ref(inp, grads, scale):
    return oracle.bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], grads["d_o"],
                      inp["initial_state"], grads["d_final_state"], inp["cu_seqlens"], scale)


def compare(got, ref, bf16):
    errs = {}
    for name, x, r in zip(NAMES, got, ref):
        if bf16 and name in ("dq", "dk", "dv"):
            errs[name] = check_close(x, r, BF16_REL, BF16_STORE, name)
        else:
            errs[name] = check_close(x, r, BF16_REL if bf16 else BWD_FP32_REL, 0.0, name)
    print("max|x - x_ref| / rms:", {k: "%.2e" % v for k, v in errs.items()})


@pytest.mark.parametrize("d_k,d_v,lens", [
    (16, 16, [5, 17, 0, 33]),
    (32, 64, [64]),
    (64, 32, [1, 15, 16, 17]),
    (128, 128, [40, 90]),
    (64, 128, [31]),
    (128, 16, [48, 2]),
])
@IMPLS
def test_bwd_fp32(cuda_lib, d_k, d_v, lens, chunked):
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=d_k, d_v=d_v, seed=600 + d_k + d_v)
    inp, grads = case(w, lens, H=2)
    compare(run_gpu(inp, grads, 0.8, chunked), run_ref(inp, grads, 0.8), bf16=False)


@pytest.mark.parametrize("base,alpha_kind,lens,H", [
    ("ckda_B1_H32_T8192_d128", None, [300, 64, 7], 2),
    ("kda_B4_H16_T2048_d128", None, [200, 1], 3),
    ("ckda_B1_H32_T8192_d128", "slow", [257], 2),
])
@IMPLS
def test_bwd_bf16(cuda_lib, base, alpha_kind, lens, H, chunked):
    kw = dict(seed=700 + sum(lens))
    if alpha_kind:
        kw["alpha_kind"] = alpha_kind
    w = custom(base, **kw)
    inp, grads = case(w, lens, H=H)
    compare(run_gpu(inp, grads, 1.0, chunked), run_ref(inp, grads, 1.0), bf16=True)


@IMPLS
def test_bwd_without_final_gradient_or_initial_state(cuda_lib, chunked):
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=32, d_v=32, seed=811)
    inp, grads = case(w, [20, 45], H=2, with_final=False, with_s0=False)
    compare(run_gpu(inp, grads, 1.0, chunked), run_ref(inp, grads, 1.0), bf16=False)


@IMPLS
def test_bwd_is_deterministic(cuda_lib, chunked):
    w = custom("ckda_B1_H32_T8192_d128", seed=812)
    inp, grads = case(w, [150, 30], H=2)
    a = run_gpu(inp, grads, 1.0, chunked)
    b = run_gpu(inp, grads, 1.0, chunked)
    for name, x, y in zip(NAMES, a, b):
        assert torch.equal(x, y), name


@IMPLS
def test_bwd_equal_length_sequences_without_cu_seqlens(cuda_lib, chunked):
    """N sequences of T tokens given by N and T alone (no cu_seqlens): the
    checkpoint slots come from n T instead of the device offsets."""
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=32, d_v=64, seed=813)
    inp, grads = case(w, [40, 40], H=2)
    d = to_dev(inp)
    g = to_dev(grads)
    got = ckda.bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], g["d_o"], d["initial_state"],
                   g["d_final_state"], N=2, T=40, scale=0.7, chunked=chunked)
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    compare(got, run_ref(inp, grads, 0.7), bf16=False)
