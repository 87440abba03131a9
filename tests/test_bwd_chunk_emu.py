"""The chunkwise backward's four per-CTA programs (csrc/ckda_bwd_split.cuh,
built from the pieces of csrc/ckda_bwd_chunk.cuh), run on the CPU through
their host executor (emu_bwd_chunk.cpp, built here with AddressSanitizer and
UBSan), against the oracle's fp64 adjoint.

This checks the programs' algebra and index arithmetic (chunks, ragged and
empty sequences, column tiles, checkpoint slots, the slot-to-chunk search,
partials) before the kernels run on a GPU; it is not a GPU parity claim. Cases and the fp32 bound
(BWD_FP32_REL * rms of the reference) are those of the GPU backward tests.
"""
import dataclasses
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_bwd_grads, make_fwd_inputs
from parity_util import check_close

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "gated_delta_rule_114_b200", "csrc")
BWD_FP32_REL = 1e-4
NAMES = ["dq", "dk", "dv", "dalpha", "dbeta", "d_initial_state"]


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("emu") / "emu_bwd_chunk")
    base = [cxx, "-std=c++17", "-O1", "-g", "-I", CSRC, os.path.join(HERE, "emu_bwd_chunk.cpp"),
            "-o", out]
    san = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]
    if subprocess.run(base[:1] + san + base[1:], capture_output=True).returncode != 0:
        subprocess.check_call(base)
    return out


def custom(base, **kw):
    return dataclasses.replace(WORKLOADS[base], **kw)


def make_case(w, lens, H, with_final=True, with_s0=True):
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
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


def f32(x):
    return np.ascontiguousarray(x.numpy() if hasattr(x, "numpy") else x, dtype=np.float32)


def run_emu(exe, tmp, inp, grads, scale, varlen=True, N=None, T=None, reverse=False):
    q = f32(inp["q"])
    Tt, H, dk = q.shape
    dv = inp["v"].shape[2]
    files = dict(q=q, k=inp["k"], v=inp["v"], alpha=inp["alpha"], beta=inp["beta"],
                 do=grads["d_o"])
    if inp["initial_state"] is not None:
        files["s0"] = inp["initial_state"]
    if grads["d_final_state"] is not None:
        files["dsf"] = grads["d_final_state"]
    for name, x in files.items():
        f32(x).tofile(os.path.join(tmp, name + ".bin"))
    cu = np.asarray(inp["cu_seqlens"], dtype=np.int32)
    if varlen:
        cu.tofile(os.path.join(tmp, "cu.bin"))
        N, T = len(cu) - 1, Tt
    env = dict(os.environ)
    env.pop("EMU_REVERSE_ITEMS", None)
    if reverse:
        env["EMU_REVERSE_ITEMS"] = "1"
    subprocess.check_call([exe, tmp, str(N), str(T), str(H), str(dk), str(dv), repr(scale),
                           str(int(varlen)), str(int("s0" in files)), str(int("dsf" in files))],
                          env=env)

    def rd(name, shape):
        return np.fromfile(os.path.join(tmp, name + ".bin"), dtype=np.float32).reshape(shape)
    return (rd("dq", (Tt, H, dk)), rd("dk", (Tt, H, dk)), rd("dv", (Tt, H, dv)),
            rd("dalpha", (Tt, H, dk)), rd("dbeta", (Tt, H)), rd("ds0", (N, H, dk, dv)))


def run_ref(inp, grads, scale):
    return oracle.bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], grads["d_o"],
                      inp["initial_state"], grads["d_final_state"], inp["cu_seqlens"], scale)


def compare(got, ref, skip_ds0=False):
    for name, x, r in zip(NAMES, got, ref):
        if name == "d_initial_state" and skip_ds0:
            continue
        check_close(x, r, BWD_FP32_REL, 0.0, name)


@pytest.mark.parametrize("d_k,d_v,lens", [
    (16, 16, [5, 17, 0, 33]),
    (16, 64, [20]),
    (32, 64, [64]),
    (64, 32, [1, 15, 16, 17]),
    (128, 128, [40, 50]),
    (128, 16, [48, 2]),
])
def test_chunk_program_fp32(emu, tmp_path, d_k, d_v, lens):
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=d_k, d_v=d_v, seed=600 + d_k + d_v)
    inp, grads = make_case(w, lens, H=2)
    compare(run_emu(emu, str(tmp_path), inp, grads, 0.8), run_ref(inp, grads, 0.8))


def test_without_final_gradient_or_initial_state(emu, tmp_path):
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=32, d_v=32, seed=811)
    inp, grads = make_case(w, [20, 45], H=2, with_final=False, with_s0=False)
    compare(run_emu(emu, str(tmp_path), inp, grads, 1.0), run_ref(inp, grads, 1.0))


def test_equal_length_sequences_without_cu_seqlens(emu, tmp_path):
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=32, d_v=64, seed=813)
    inp, grads = make_case(w, [40, 40], H=2)
    got = run_emu(emu, str(tmp_path), inp, grads, 0.7, varlen=False, N=2, T=40)
    compare(got, run_ref(inp, grads, 0.7))


@pytest.mark.parametrize("kind", ["zero", "sign", "mixed"])
def test_degenerate_gates(emu, tmp_path, kind):
    """alpha = 0 everywhere, alpha = +-1 everywhere, and a mix of exact 0,
    +-1 and tiny entries: the gate gradient takes no logarithm or division."""
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=32, d_v=32, seed=820)
    inp, grads = make_case(w, [37, 9], H=2)
    rng = np.random.default_rng(5)
    shape = tuple(inp["alpha"].shape)
    if kind == "zero":
        a = np.zeros(shape)
    elif kind == "sign":
        a = np.sign(rng.normal(size=shape))
    else:
        a = np.asarray(inp["alpha"], dtype=np.float64)
        u = rng.uniform(size=shape)
        a = np.where(u < 0.1, np.sign(rng.normal(size=shape)), a)
        a = np.where((u >= 0.1) & (u < 0.2), 0.0, a)
        a = np.where((u >= 0.2) & (u < 0.25), 1e-6 * rng.normal(size=shape), a)
    inp["alpha"] = torch.from_numpy(a.astype(np.float32))
    compare(run_emu(emu, str(tmp_path), inp, grads, 1.0), run_ref(inp, grads, 1.0))


def test_items_of_a_phase_are_independent(emu, tmp_path):
    """Every phase's items in reverse order give bit-identical gradients: no
    item reads what another item of its phase writes (the GPU runs them at
    once)."""
    w = custom("ckda_B1_H32_T8192_d128", dtype="f32", d_k=64, d_v=64, seed=830)
    inp, grads = make_case(w, [37, 16, 5], H=2)
    fwd = run_emu(emu, str(tmp_path), inp, grads, 0.9)
    rev = run_emu(emu, str(tmp_path), inp, grads, 0.9, reverse=True)
    for name, x, y in zip(NAMES, fwd, rev):
        assert np.array_equal(x, y), name


@pytest.fixture(scope="module")
def slot_map(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("slots") / "emu_slot_map")
    subprocess.check_call([cxx, "-std=c++17", "-O1", "-I", CSRC,
                           os.path.join(HERE, "emu_slot_map.cpp"), "-o", out])
    return out


@pytest.mark.parametrize("seed", range(6))
def test_every_slot_finds_its_chunk(slot_map, seed):
    """slot_chunk, the per-chunk grids' map from checkpoint slot to (sequence,
    chunk), against an enumeration: every chunk's slot maps back to it, and
    every other slot is one the kernels skip (no sequence, or past its last
    chunk), so no chunk runs twice and none is missed."""
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 9))
    lens = rng.choice([0, 1, 15, 16, 17, 31, 32, 33, 64, 100], size=N)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    cases = [(N, 0, list(cu)), (N, int(lens[0]), None)]  # varlen; N equal sequences
    for n_seq, T, offsets in cases:
        if offsets is None:
            offsets = [i * T for i in range(n_seq + 1)]
        args = [slot_map, str(n_seq), str(T)] + ([str(c) for c in offsets] if T == 0 else [])
        out = subprocess.run(args, check=True, capture_output=True, text=True).stdout.split("\n")
        got = {int(g): (int(n), int(ci), int(ok))
               for g, n, ci, ok in (line.split() for line in out if line)}
        want = {}
        for n in range(n_seq):
            b, e = offsets[n], offsets[n + 1]
            for ci in range((e - b + 15) // 16):
                want[b // 16 + n + ci] = (n, ci)
        assert len(got) == offsets[-1] // 16 + n_seq
        assert all(g in got for g in want)  # every chunk's slot is inside the grid
        for g, (n, ci, ok) in got.items():
            nck = (offsets[n + 1] - offsets[n] + 15) // 16 if 0 <= n < n_seq else 0
            runs = bool(ok) and ci < nck
            assert runs == (g in want), (g, n, ci, ok)
            if runs:
                assert (n, ci) == want[g], g
