"""The complex-phase gate's chunked forward programs
(csrc/ckda_complex_chunk.cuh), run on the CPU through their host executor
(emu_complex_chunk.cpp, built here with AddressSanitizer and UBSan), against
the oracle's complex128 token recurrence (oracle.fwd_complex, pinned in
test_oracle_complex.py).

This checks the programs' algebra and index arithmetic (chunks, ragged and
empty sequences, column tiles, checkpoint slots) before the kernels run on a
GPU; it is not a GPU parity claim. Cases follow the GPU tests of
ckda_fwd_complex, with the fp32 check-mode bound 1e-5 * rms.
"""
import dataclasses
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_complex_inputs
from parity_util import FP32_REL, check_close

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "gated_delta_rule_114_b200", "csrc")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("emu") / "emu_complex_chunk")
    base = [cxx, "-std=c++17", "-O1", "-g", "-I", CSRC,
            os.path.join(HERE, "emu_complex_chunk.cpp"), "-o", out]
    san = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]
    if subprocess.run(base[:1] + san + base[1:], capture_output=True).returncode != 0:
        subprocess.check_call(base)
    return out


def custom(**kw):
    return dataclasses.replace(WORKLOADS["ckda_B1_H32_T8192_d128"], dtype="f32", **kw)


def lens_cu(lens):
    return torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))


def c64(x):
    """complex tensor -> interleaved float32 (real, imaginary) array"""
    return np.ascontiguousarray(torch.view_as_real(x.to(torch.complex64)).numpy())


def run_emu(exe, tmp, inp, scale, with_s0=True, varlen=True, N=None, T=None, reverse=False):
    Tt, H, dk = inp["q"].shape
    dv = inp["v"].shape[2]
    for name in ("q", "k", "v"):
        c64(inp[name]).tofile(os.path.join(tmp, name + ".bin"))
    for name in ("alpha", "theta", "beta"):
        np.ascontiguousarray(inp[name].numpy(), dtype=np.float32).tofile(
            os.path.join(tmp, name + ".bin"))
    if with_s0:
        c64(inp["initial_state"]).tofile(os.path.join(tmp, "s0.bin"))
    cu = np.asarray(inp["cu_seqlens"], dtype=np.int32)
    if varlen:
        cu.tofile(os.path.join(tmp, "cu.bin"))
        N, T = len(cu) - 1, Tt
    env = dict(os.environ)
    env.pop("EMU_REVERSE_ITEMS", None)
    if reverse:
        env["EMU_REVERSE_ITEMS"] = "1"
    subprocess.check_call([exe, tmp, str(N), str(T), str(H), str(dk), str(dv), repr(scale),
                           str(int(varlen)), str(int(with_s0))], env=env)
    o = np.fromfile(os.path.join(tmp, "o.bin"), dtype=np.float32).reshape(Tt, H, dv, 2)
    sf = np.fromfile(os.path.join(tmp, "sf.bin"), dtype=np.float32).reshape(N, H, dk, dv, 2)
    return o, sf


def check(got, inp, scale, with_s0=True):
    o_ref, sf_ref = oracle.fwd_complex(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["theta"],
                                       inp["beta"], inp["initial_state"] if with_s0 else None,
                                       inp["cu_seqlens"], scale)
    for x, r, name in ((got[0], o_ref, "o"), (got[1], sf_ref, "final_state")):
        check_close(x, np.stack([r.real, r.imag], axis=-1), FP32_REL, 0.0, name)


@pytest.mark.parametrize("d_k,d_v,lens,ranges", [
    (16, 16, [5, 17, 0, 33], "sfda"),
    (64, 32, [64, 1, 40], "ckda"),
    (128, 128, [100, 37], "sfda"),
    (32, 64, [90], "ckda"),
    (16, 64, [15, 16, 17], "ckda"),
])
def test_chunked_complex_forward(emu, tmp_path, d_k, d_v, lens, ranges):
    w = custom(d_k=d_k, d_v=d_v, seed=900 + d_k + d_v)
    inp = make_complex_inputs(w, lens_cu(lens), H=2, ranges=ranges)
    check(run_emu(emu, str(tmp_path), inp, 0.8), inp, 0.8)


def test_without_initial_state(emu, tmp_path):
    w = custom(d_k=32, d_v=32, seed=931)
    inp = make_complex_inputs(w, lens_cu([20, 45]), H=2)
    check(run_emu(emu, str(tmp_path), inp, 1.0, with_s0=False), inp, 1.0, with_s0=False)


def test_equal_lengths_without_cu_seqlens(emu, tmp_path):
    w = custom(d_k=64, d_v=64, seed=932)
    inp = make_complex_inputs(w, lens_cu([33, 33]), H=2)
    check(run_emu(emu, str(tmp_path), inp, 1.0, varlen=False, N=2, T=33), inp, 1.0)


@pytest.mark.parametrize("kind", ["zero", "unit"])
def test_degenerate_gates(emu, tmp_path, kind):
    """alpha = 0 (every gate product through a zero is exactly 0) and |alpha| =
    1 (pure rotations, nothing decays over the chunk)."""
    w = custom(d_k=32, d_v=32, seed=940)
    inp = make_complex_inputs(w, lens_cu([37, 9]), H=2, ranges="ckda")
    a = inp["alpha"].clone()
    if kind == "zero":
        a[::3] = 0.0
    else:
        a = torch.sign(a)
    inp["alpha"] = a.contiguous()
    check(run_emu(emu, str(tmp_path), inp, 1.0), inp, 1.0)


def test_items_of_a_phase_are_independent(emu, tmp_path):
    """Every phase's items in reverse order give bit-identical outputs: no item
    reads what another item of its phase writes (the GPU runs them at once)."""
    w = custom(d_k=64, d_v=64, seed=950)
    inp = make_complex_inputs(w, lens_cu([37, 16, 5]), H=2, ranges="ckda")
    fwd = run_emu(emu, str(tmp_path), inp, 0.9)
    rev = run_emu(emu, str(tmp_path), inp, 0.9, reverse=True)
    assert np.array_equal(fwd[0], rev[0]) and np.array_equal(fwd[1], rev[1])
