"""Run one kernel of the library on one workload a few times (for profilers).

    python -m gated_delta_rule_114_b200.run_case --case prefill [--T 4096] [--iters 3]
    python -m gated_delta_rule_114_b200.run_case --case decode [--N 64] [--iters 3]
    python -m gated_delta_rule_114_b200.run_case --case bwd [--T 2048] [--iters 2] [--chunked]
    python -m gated_delta_rule_114_b200.run_case --case complex [--T 2048] [--iters 2] [--chunked]

The prefill case uses the CKDA long-prefill recipe (H=32, d=128, bf16 I/O,
CKDA gates, random initial state) with T tokens per head; the decode case
uses the decode recipe with N sequences. It prints nothing but a line with
the shapes; it is meant to be wrapped by a profiler, not to time anything.
The bwd case runs the backward pass on the prefill recipe with seeded
upstream gradients; the complex case the complex-phase gate on complex64
inputs of the same shape. --chunked selects the chunked entry point of either.
"""
from __future__ import annotations

import argparse

import torch

from gated_delta_rule_114_b200 import ckda
from gated_delta_rule_114_b200.inputs import (WORKLOADS, make_bwd_grads,
                                              make_complex_inputs,
                                              make_decode_state,
                                              make_decode_tokens,
                                              make_fwd_inputs)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["prefill", "decode", "bwd", "complex"], default="prefill")
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--N", type=int, default=64)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--chunked", action="store_true",
                    help="bwd and complex cases: the chunked entry point")
    args = ap.parse_args()
    ckda.load()
    if args.case == "prefill":
        w = WORKLOADS["ckda_B1_H32_T8192_d128"]
        cu = torch.tensor([0, args.T], dtype=torch.int32)
        inp = make_fwd_inputs(w, cu_seqlens=cu, H=args.H)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        for _ in range(args.iters):
            ckda.fwd_chunked(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                             d["initial_state"], d["cu_seqlens"], chunk=w.chunk)
        shape = "T=%d H=%d d=128" % (args.T, args.H)
    elif args.case == "bwd":
        w = WORKLOADS["ckda_B1_H32_T8192_d128"]
        cu = torch.tensor([0, args.T], dtype=torch.int32)
        inp = make_fwd_inputs(w, cu_seqlens=cu, H=args.H)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        g = {k: v.cuda() for k, v in make_bwd_grads(w, args.T, args.H, 1).items()}
        for _ in range(args.iters):
            ckda.bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], g["d_o"],
                     d["initial_state"], g["d_final_state"], cu_seqlens=d["cu_seqlens"],
                     chunked=args.chunked)
        shape = "T=%d H=%d d=128" % (args.T, args.H)
    elif args.case == "complex":
        w = WORKLOADS["ckda_B1_H32_T8192_d128"]
        cu = torch.tensor([0, args.T], dtype=torch.int32)
        c = {k: v.cuda() for k, v in make_complex_inputs(w, cu, args.H).items()}
        for _ in range(args.iters):
            ckda.fwd_complex(c["q"], c["k"], c["v"], c["alpha"], c["theta"], c["beta"],
                             c["initial_state"], cu_seqlens=c["cu_seqlens"], chunked=args.chunked)
        shape = "T=%d H=%d d=128 complex64" % (args.T, args.H)
    else:
        w = WORKLOADS["decode_N256_H32_d128"]
        state = make_decode_state(w, N=args.N).cuda()
        tok = {k: v.cuda() for k, v in make_decode_tokens(w, 0, N=args.N).items()}
        for _ in range(args.iters):
            ckda.decode_step(tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], state)
        shape = "N=%d H=32 d=128" % args.N
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    print("run_case %s %s iters=%d ok" % (args.case, shape, args.iters))


if __name__ == "__main__":
    main()
