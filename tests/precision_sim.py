"""Rounding model of the tensor-core forward: which products can take bf16 operands?

A CPU restatement of the chunk-WY data flow of the tensor-core path (64-token
chunks, Grams factored at the 16-token sub-block and 4-token group boundaries,
T = (I + A)^-1, the two WY products, then the state chain) in fp64, rounding
the operands of each tensor-core product to a chosen format (fp32, tf32 with
round-to-nearest-away as cvt.rna.tf32.f32 does, tf32 cut off (what an MMA
reading an unrounded fp32 value uses), or bf16 round-to-nearest-even)
and keeping the accumulations exact. It compares o and the final state with
the fp64 token oracle on the CKDA long-prefill distribution. It is neither the
oracle nor the CUDA path: it only tells which operand precision each product
needs to stay inside the 1e-2 * rms(o) bound (Complex KDA: the output tolerance
of the bf16 path).

    python tests/precision_sim.py [--T 2048] [--H 8]

prints, per variant, max|o - o_ref| / rms(o_ref) before the bf16 store, the
excess over the store allowance 2^-8 |o_ref| after it, and the final state's
max error / rms.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_fwd_inputs  # noqa: E402


def rnd(x, kind):
    if kind == "f64":
        return x
    if kind == "f32":
        return x.astype(np.float32).astype(np.float64)
    if kind == "tf32":  # keep 10 mantissa bits, ties away from zero
        b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
        b = (b + 0x1000) & 0xFFFFE000
        return b.astype(np.uint32).view(np.float32).astype(np.float64)
    if kind == "tf32t":  # keep 10 mantissa bits, the rest cut off
        b = x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
        return b.view(np.float32).astype(np.float64)
    if kind == "bf16":
        return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    raise ValueError(kind)


def chunk(S, q, k, v, al, be, P):
    """One 64-token chunk for H heads at once; P maps product -> operand format."""
    H, L, dk = q.shape
    G = np.zeros((H, L, L, dk))
    for j in range(L):
        g = np.ones((H, dk))
        G[:, j, j] = g
        for i in range(j + 1, L):
            g = g * al[:, i]
            G[:, i, j] = g
    A = np.zeros((H, L, L))
    M = np.zeros((H, L, L))
    for i in range(L):
        for j in range(i + 1):
            if j // 16 < i // 16:        # different sub-blocks: one product
                r, fmt = 16 * (i // 16) - 1, P["gram"]
            elif j // 4 < i // 4:        # same sub-block, different groups
                r, fmt = 4 * (i // 4) - 1, P["gram"]
            else:                        # same 4-token group: CUDA cores, fp32
                r, fmt = None, None
            if r is None:
                gk = G[:, i, j] * k[:, j]
                M[:, i, j] = np.sum(q[:, i] * gk, -1)
                if j < i:
                    A[:, i, j] = be[:, i] * np.sum(k[:, i] * gk, -1)
                continue
            rr = rnd(k[:, j] * G[:, r, j], fmt)
            M[:, i, j] = np.sum(rnd(q[:, i] * G[:, i, r], fmt) * rr, -1)
            if j < i:
                A[:, i, j] = be[:, i] * np.sum(rnd(k[:, i] * G[:, i, r], fmt) * rr, -1)
    A, M = rnd(A, "f32"), rnd(M, "f32")
    T = rnd(np.linalg.inv(np.eye(L)[None] + A), "f32")
    gam = np.cumprod(al, axis=1)
    sig = np.stack([G[:, L - 1, j] for j in range(L)], 1)
    MT = rnd(M, P["mt"]) @ rnd(T, P["mt"])
    bK = rnd(be[..., None] * gam * k, P["wy"])
    bV = rnd(be[..., None] * v, P["wy"])
    Tq, MTq = rnd(T, P["wy"]), rnd(MT, P.get("mtq", P["wy"]))
    W, Ut, MW, MUt = Tq @ bK, Tq @ bV, MTq @ bK, MTq @ bV
    Qt = gam * q - MW
    Sq = rnd(S, P["state"])
    U = Ut - rnd(W, P["scan"]) @ Sq
    O = rnd(Qt, P["scan"]) @ Sq + MUt
    S_new = gam[:, -1][..., None] * S + np.swapaxes(rnd(sig * k, P["scan"]), 1, 2) @ rnd(U, P["state"])
    return O, rnd(S_new, "f32")


def run(P, T, H, seed):
    w = dataclasses.replace(WORKLOADS["ckda_B1_H32_T8192_d128"], seed=seed)
    cu = torch.tensor([0, T], dtype=torch.int32)
    inp = make_fwd_inputs(w, cu_seqlens=cu, H=H)
    tr = {key: inp[key].double().numpy().transpose(1, 0, 2) for key in ("q", "k", "v", "alpha")}
    be = inp["beta"].double().numpy().T
    S = inp["initial_state"][0].double().numpy()
    o_ref, sf_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               inp["initial_state"], cu)
    o = np.zeros((H, T, tr["v"].shape[2]))
    for s in range(0, T, 64):
        e = s + 64
        o[:, s:e], S = chunk(S, tr["q"][:, s:e], tr["k"][:, s:e], tr["v"][:, s:e],
                             tr["alpha"][:, s:e], be[:, s:e], P)
    o = o.transpose(1, 0, 2)
    r = np.sqrt(np.mean(o_ref ** 2))
    ob = rnd(o, "bf16")
    return (np.abs(o - o_ref).max() / r,
            (np.abs(ob - o_ref) - 2.0 ** -8 * np.abs(o_ref)).max() / r,
            np.abs(S - sf_ref[0]).max() / np.sqrt(np.mean(sf_ref ** 2)))


VARIANTS = {
    "fp64 operands (model check)": dict(gram="f64", mt="f64", wy="f64", scan="f64", state="f64"),
    "tf32 everywhere (the kernels)": dict(gram="tf32", mt="tf32", wy="tf32", scan="tf32", state="tf32"),
    "bf16 Gram operands": dict(gram="bf16", mt="tf32", wy="tf32", scan="tf32", state="tf32"),
    "bf16 [M;I] x T": dict(gram="tf32", mt="bf16", wy="tf32", scan="tf32", state="tf32"),
    "[MT;T] truncated as D5's A operand": dict(gram="tf32", mt="tf32", wy="tf32", mtq="tf32t",
                                               scan="tf32", state="tf32"),
    "bf16 WY product": dict(gram="tf32", mt="tf32", wy="bf16", scan="tf32", state="tf32"),
    "bf16 chain A operands, tf32 S and U": dict(gram="tf32", mt="tf32", wy="tf32", scan="bf16", state="tf32"),
    "bf16 chain (A and S, U)": dict(gram="tf32", mt="tf32", wy="tf32", scan="bf16", state="bf16"),
    "bf16 everywhere": dict(gram="bf16", mt="bf16", wy="bf16", scan="bf16", state="bf16"),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--H", type=int, default=8)
    ap.add_argument("--seed", type=int, default=1003)
    args = ap.parse_args()
    print("T=%d H=%d, CKDA long-prefill distribution (seed %d)" % (args.T, args.H, args.seed))
    print("%-38s %10s %12s %10s" % ("variant", "o pre-store", "store excess", "state"))
    for name, P in VARIANTS.items():
        t0 = time.time()
        e = run(P, args.T, args.H, args.seed)
        print("%-38s %10.2e %12.2e %10.2e  (%.0f s)" % (name, *e, time.time() - t0), flush=True)


if __name__ == "__main__":
    main()
