"""Benchmark of the CKDA hot path on B200: chunked prefill forward + decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0. A "step" is one chunked forward (every step of the
chunkwise path: load, gate cumulant, Grams, UT solve, WY factors, state
propagation and output) over the CKDA long-prefill batch (B=1, H=32,
T=8192, d_k=d_v=128, bf16 I/O, fp32 state), inputs resident in HBM. The decode
step (256 sequences x 32 heads, fp32 state in HBM) is timed in the same run
and reported under "decode". N>1 (torchrun, one rank per GPU): every rank runs
its own copy of the batch (heads and sequences are independent, so no
collective sits on the data path); value = all ranks' tokens / max time.

--impl reference runs the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (rank 0 only).

    python bench.py --case prefill|decode|bwd|complex [--T 4096] [--H 32] [--N 64]
                    [--iters 3] [--chunked]

runs one entry point a few times on one workload and times nothing (a
command for a profiler to wrap): prefill uses the CKDA long-prefill recipe
with T tokens per head, decode the decode recipe with N sequences, bwd the
backward pass on the prefill recipe with seeded upstream gradients, complex
the complex-phase gate on complex64 inputs of the same shape; --chunked
selects the chunked entry point of bwd or complex.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_114_b200 import ckda  # noqa: E402
from gated_delta_rule_114_b200.inputs import (WORKLOADS, make_bwd_grads,  # noqa: E402
                                              make_complex_inputs,
                                              make_decode_state,
                                              make_decode_tokens,
                                              make_fwd_inputs,
                                              make_gated_fwd_inputs)

METRIC = ("CKDA prefill tokens/s (H=32, d=128, T=8192) + % bf16 roofline; "
          "decode tok/s, HBM GB/s")
PREFILL = "ckda_B1_H32_T8192_d128"
DECODE = "decode_N256_H32_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def esize(dt):
    return 2 if dt == torch.bfloat16 else 4


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the current kernels, scaled by the units processed; the
# capture, its command and the scaling are in profiles/. Set to None whenever
# a kernel changes after its capture.
NCU_TRAFFIC = {
    # prep + scan at T=2048, H=32 (1024 chunk-heads): 193.3 + 178.5 MB, x4 for T=8192
    "prefill": 4 * 371.8e6,
    # N=64 (2048 pairs): 214.8 MB, x4 for N=256
    "decode": 4 * 214.8e6,
    # token-serial backward (both kernels) at T=512, H=32: 356.3 MB, x16 for T=8192
    "backward": 16 * 356.3e6,
    # chunked backward (prep, two scans, gradients) at T=2048, H=32: 2021.9 MB,
    # x4 for T=8192
    "backward_chunked": 4 * 2021.9e6,
}


def prefill_bytes(inp) -> int:
    """Algorithmic HBM bytes of one forward: every input read once, every
    output written once (q, k, v, alpha, beta, o per token-head; states)."""
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[2]
    es = esize(inp["q"].dtype)
    per_th = (2 * dk + dv) * es + dk * 4 + 4 + dv * es
    N = inp["cu_seqlens"].numel() - 1
    st = N * H * dk * dv * 4
    return T * H * per_th + (st if inp["initial_state"] is not None else 0) + st


def prefill_flops(inp, C=64) -> float:
    """Useful flops of the chunked form: per chunk 2.5 C^2 d + 3 C d^2 + C^3/6
    multiply-adds (Grams, WY factors, state/output contractions, UT solve)."""
    T, H, d = inp["q"].shape
    cu = inp["cu_seqlens"].tolist()
    mac = 0.0
    for n in range(len(cu) - 1):
        L = cu[n + 1] - cu[n]
        full, rem = divmod(L, C)
        for c in [C] * full + ([rem] if rem else []):
            mac += 2.5 * c * c * d + 3 * c * d * d + c ** 3 / 6.0
    return 2.0 * mac * H


def prefill_gated_bytes(inp) -> int:
    """Algorithmic HBM bytes of one forward with the fused input prologue:
    q, k_raw, v, a_logit (I/O dtype), c_logit (fp32), o per token-head; states."""
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[2]
    es = esize(inp["q"].dtype)
    per_th = (3 * dk + dv) * es + 4 + dv * es
    N = inp["cu_seqlens"].numel() - 1
    st = N * H * dk * dv * 4
    return T * H * per_th + (st if inp["initial_state"] is not None else 0) + st


def bwd_bytes(inp) -> int:
    """Algorithmic HBM bytes of one backward call: the forward's inputs and
    do read once, dq, dk, dv, dalpha, dbeta written once per token-head;
    initial state and final-state gradient read, initial-state gradient
    written once per (sequence, head)."""
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[2]
    es = esize(inp["q"].dtype)
    per_th = ((2 * dk + dv) * es + dk * 4 + 4 + dv * es) + ((2 * dk + dv) * es + dk * 4 + 4)
    N = inp["cu_seqlens"].numel() - 1
    return T * H * per_th + 3 * N * H * dk * dv * 4


def complex_bytes(T, H, N, dk, dv) -> int:
    """Algorithmic HBM bytes of one complex-phase-gate forward: q, k, v, o
    complex64, alpha, theta, beta fp32 per token-head; initial and final
    complex64 states per (sequence, head)."""
    return T * H * ((2 * dk + 2 * dv) * 8 + 2 * dk * 4 + 4) + 2 * N * H * dk * dv * 8


def decode_bytes(N, H, dk, dv, dt) -> int:
    es = esize(dt)
    return N * H * (2 * dk * dv * 4 + (2 * dk + dv) * es + dk * 4 + 4 + dv * es)


class ClockSampler:
    """Samples SM clock and throttle reasons while the timed region runs."""

    REASONS = {  # NVML clocks-event-reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.02):
        self.index = index
        self.period = period
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def time_loop(fn, steps: int, warmup: int, stream, barrier=None):
    """W untimed calls, then K calls between CUDA events on `stream`."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return start.elapsed_time(end) / steps  # ms per step


def cpu_baseline_prefill(w, inp_cpu, target_s=12.0):
    """Oracle (as it stands) on a bounded sample: the first h heads of the
    prefill batch, h grown until one run takes about target_s seconds."""
    import oracle
    cores = oracle.max_threads()
    T = inp_cpu["q"].shape[0]
    H = inp_cpu["q"].shape[1]
    h = 1
    while True:
        sub = {key: inp_cpu[key][:, :h].contiguous() for key in
               ("q", "k", "v", "alpha", "beta")}
        s0 = inp_cpu["initial_state"][:, :h].contiguous()
        t0 = time.perf_counter()
        oracle.fwd(sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"], s0,
                   inp_cpu["cu_seqlens"])
        dt = time.perf_counter() - t0
        if dt >= target_s / 3 or h >= H:
            break
        h = min(H, max(h + 1, int(h * target_s / max(dt, 1e-3))))
    tok_heads = T * h
    return {"value": tok_heads / dt / H, "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": ("fp64 token-by-token oracle on %d of %d heads x %d tokens "
                       "(%d token-heads, %.2f s); tokens/s = token-heads/s / %d heads"
                       % (h, H, T, tok_heads, dt, H))}


def chunked_legs(args, w, inp_cpu, T_total, H, N, dk, dv, stream, pk, world):
    """The chunked backward and complex-gate entry points on the bench's shape,
    timed on this rank alone (no collective), after every other leg. Any
    failure is recorded in the returned dict instead of ending the run."""
    out = {}
    try:
        dev = {key: (val.cuda() if isinstance(val, torch.Tensor) else val)
               for key, val in inp_cpu.items()}
        if args.bwd_impl != "chunked":
            bg = make_bwd_grads(w, T_total, H, N)
            bdo, bdsf = bg["d_o"].cuda(), bg["d_final_state"].cuda()
            bout = [torch.empty_like(dev["q"]), torch.empty_like(dev["k"]),
                    torch.empty_like(dev["v"]), torch.empty_like(dev["alpha"]),
                    torch.empty_like(dev["beta"]),
                    torch.empty((N, H, dk, dv), dtype=torch.float32, device="cuda")]
            bws = torch.empty(ckda.ckda_bwd_workspace_bytes(N, T_total, H, dk, dv, True, True),
                              dtype=torch.uint8, device="cuda")

            def bstep():
                ckda.ckda_bwd(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"],
                              dev["initial_state"], bdo, bdsf, *bout, dev["cu_seqlens"], None,
                              stream=stream, workspace=bws, chunked=True)

            ms = time_loop(bstep, args.bwd_steps, 3, stream)
            if ckda.ckda_last_error() != ckda.CKDA_OK:
                raise RuntimeError("kernel reported an error")
            nb = bwd_bytes(inp_cpu)
            out["backward_chunked"] = {
                "entry_point": "ckda_bwd_chunked", "ms_per_step": ms,
                "tokens_per_s": T_total / (ms / 1e3), "steps": args.bwd_steps, "warmup": 3,
                "roofline": {"bound": "hbm", "achieved": nb / (ms / 1e3) / 1e9,
                             "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": nb / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "traffic": None,
                             "algorithmic_bytes_per_launch": nb},
                "timing": "this rank alone", "gpu_launches": 4 * args.bwd_steps}
            del bws, bout, bdo, bdsf
        if args.complex_impl != "chunked":
            cin = {key: val.cuda() for key, val in
                   make_complex_inputs(w, inp_cpu["cu_seqlens"], H).items()}
            co = torch.empty((T_total, H, dv), dtype=torch.complex64, device="cuda")
            csf = torch.empty((N, H, dk, dv), dtype=torch.complex64, device="cuda")
            cws = torch.empty(ckda.ckda_fwd_complex_chunked_workspace_bytes(N, T_total, H, dk, dv,
                                                                             True),
                              dtype=torch.uint8, device="cuda")

            def cstep():
                ckda.ckda_fwd_complex(cin["q"], cin["k"], cin["v"], cin["alpha"], cin["theta"],
                                      cin["beta"], cin["initial_state"], csf, co,
                                      cin["cu_seqlens"], None, stream=stream, chunked=True,
                                      workspace=cws)

            ms = time_loop(cstep, args.complex_steps, 3, stream)
            if ckda.ckda_last_error() != ckda.CKDA_OK:
                raise RuntimeError("kernel reported an error")
            nb = complex_bytes(T_total, H, N, dk, dv)
            out["complex_gate_chunked"] = {
                "entry_point": "ckda_fwd_complex_chunked", "ms_per_step": ms,
                "tokens_per_s": T_total / (ms / 1e3), "steps": args.complex_steps, "warmup": 3,
                "roofline": {"bound": "hbm", "achieved": nb / (ms / 1e3) / 1e9,
                             "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": nb / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "traffic": None,
                             "algorithmic_bytes_per_launch": nb},
                "timing": "this rank alone", "gpu_launches": 2 * args.complex_steps}
            del cws, cin, co, csf
    except Exception as e:  # recorded, not fatal: these legs come after every other one
        out["chunked_legs_error"] = "%s: %s" % (type(e).__name__, e)
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = WORKLOADS[PREFILL]
    inp = make_fwd_inputs(w)
    cores = oracle.max_threads()
    T, H = inp["q"].shape[:2]
    # one head per host core per step (the oracle runs its (sequence, head)
    # pairs in parallel): a bounded sample that keeps every core busy
    h = max(1, min(H, cores))
    sub = {key: inp[key][:, :h].contiguous() for key in ("q", "k", "v", "alpha", "beta")}
    s0 = inp["initial_state"][:, :h].contiguous()

    def step():
        oracle.fwd(sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"], s0,
                   inp["cu_seqlens"])

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = T * h / (ms / 1e3) / H
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": PREFILL, "global_batch": 1, "seq_len": T,
                   "heads": H, "d_k": 128, "d_v": 128, "chunk": 64,
                   "sample_heads_per_step": h},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": "fp64 oracle on %d of %d heads x %d tokens per step; "
                                   "tokens/s = token-heads/s / %d heads" % (h, H, T, H)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_case(args):
    """One entry point, args.iters calls, no timing (see the module doc)."""
    ckda.load()
    T, H = args.T, args.H
    if args.case in ("prefill", "bwd", "complex"):
        w = WORKLOADS[PREFILL]
        cu = torch.tensor([0, T], dtype=torch.int32)
    if args.case == "prefill":
        inp = make_fwd_inputs(w, cu_seqlens=cu, H=H)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        for _ in range(args.iters):
            ckda.fwd_chunked(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                             d["initial_state"], d["cu_seqlens"], chunk=w.chunk)
        shape = "T=%d H=%d d=128" % (T, H)
    elif args.case == "bwd":
        inp = make_fwd_inputs(w, cu_seqlens=cu, H=H)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        g = {k: v.cuda() for k, v in make_bwd_grads(w, T, H, 1).items()}
        for _ in range(args.iters):
            ckda.bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], g["d_o"],
                     d["initial_state"], g["d_final_state"], cu_seqlens=d["cu_seqlens"],
                     chunked=args.chunked)
        shape = "T=%d H=%d d=128" % (T, H)
    elif args.case == "complex":
        c = {k: v.cuda() for k, v in make_complex_inputs(w, cu, H).items()}
        for _ in range(args.iters):
            ckda.fwd_complex(c["q"], c["k"], c["v"], c["alpha"], c["theta"], c["beta"],
                             c["initial_state"], cu_seqlens=c["cu_seqlens"], chunked=args.chunked)
        shape = "T=%d H=%d d=128 complex64" % (T, H)
    else:
        w = WORKLOADS[DECODE]
        state = make_decode_state(w, N=args.N).cuda()
        tok = {k: v.cuda() for k, v in make_decode_tokens(w, 0, N=args.N).items()}
        for _ in range(args.iters):
            ckda.decode_step(tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], state)
        shape = "N=%d H=32 d=128" % args.N
    torch.cuda.synchronize()
    if ckda.ckda_last_error() != ckda.CKDA_OK:
        raise RuntimeError("kernel reported an error")
    print("case %s %s iters=%d ok" % (args.case, shape, args.iters))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--bwd-steps", type=int, default=5)
    ap.add_argument("--bwd-impl", default="chunked", choices=["serial", "chunked"],
                    help="backward entry point: ckda_bwd (token-serial) or ckda_bwd_chunked")
    ap.add_argument("--complex-steps", type=int, default=5)
    ap.add_argument("--complex-impl", default="chunked", choices=["serial", "chunked"],
                    help="complex-gate entry point: ckda_fwd_complex (token-serial) or "
                         "ckda_fwd_complex_chunked")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-chunked-legs", action="store_true",
                    help="skip the extra timing of the chunked backward and complex paths")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["prefill", "decode", "bwd", "complex"], default=None,
                    help="run one entry point --iters times for a profiler; no timing")
    ap.add_argument("--T", type=int, default=4096, help="--case: tokens per head")
    ap.add_argument("--H", type=int, default=32, help="--case: heads")
    ap.add_argument("--N", type=int, default=64, help="--case decode: sequences")
    ap.add_argument("--iters", type=int, default=3, help="--case: calls")
    ap.add_argument("--chunked", action="store_true",
                    help="--case bwd / complex: the chunked entry point")
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    barrier = (lambda: dist.barrier()) if dist else None
    ckda.load()
    stream = torch.cuda.current_stream()
    pk = peaks()

    # ---------------- prefill (the headline step)
    w = WORKLOADS[PREFILL]
    inp_cpu = make_fwd_inputs(w)
    dev = {key: (val.cuda() if isinstance(val, torch.Tensor) else val)
           for key, val in inp_cpu.items()}
    T_total, H, dk = dev["q"].shape
    dv = dev["v"].shape[2]
    N = dev["cu_seqlens"].numel() - 1
    o = torch.empty((T_total, H, dv), dtype=dev["q"].dtype, device="cuda")
    sf = torch.empty((N, H, dk, dv), dtype=torch.float32, device="cuda")
    ws_bytes = ckda.ckda_fwd_workspace_bytes(N, T_total, H, dk, dv, w.chunk,
                                             True, dev["q"].dtype)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")

    def prefill():
        ckda.ckda_fwd_chunked(dev["q"], dev["k"], dev["v"], dev["alpha"],
                              dev["beta"], dev["initial_state"], sf, o,
                              dev["cu_seqlens"], None, chunk=w.chunk,
                              stream=stream, workspace=ws)

    with ClockSampler(local) as clk:
        ms = time_loop(prefill, args.steps, args.warmup, stream, barrier)
    if ckda.ckda_last_error() != ckda.CKDA_OK:
        raise RuntimeError("kernel reported an error")
    ms_max = ms
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    tokens = T_total * world
    value = tokens / (ms_max / 1e3)
    nbytes = prefill_bytes(inp_cpu)
    flops = prefill_flops(inp_cpu, w.chunk)
    achieved = nbytes / (ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                "traffic": NCU_TRAFFIC["prefill"], "peak_source": pk["source"],
                "algorithmic_bytes_per_launch": nbytes,
                # every tensor-core product is tf32: its peak is the measured bf16
                # peak times the nominal tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s)
                "tensor": {"achieved_tflops": flops / (ms / 1e3) / 1e12,
                           "peak_tflops": pk["bf16_tflops"] * 1.1 / 2.25,
                           "peak_source": "measured bf16 x 1.1/2.25 (tf32 operands)",
                           "frac": flops / (ms / 1e3) / 1e12 / (pk["bf16_tflops"] * 1.1 / 2.25),
                           "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / pk["bf16_tflops"],
                           "useful_flops_per_launch": flops}}

    # ---------------- end to end through the C ABI with host buffers. Every
    # step copies its inputs from pinned host memory, runs the forward and
    # copies o and the final state back. Copies in, compute and copies out sit
    # on three streams with two device buffer sets, so step i + 1's inputs
    # cross the link while step i computes and step i - 1's outputs return
    # (the link's two directions and the GPU work overlap, as in a serving
    # loop); the timed region is every step's copies and compute.
    pinned = {key: (val.pin_memory() if isinstance(val, torch.Tensor) else val)
              for key, val in inp_cpu.items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    sf_host = torch.empty(sf.shape, dtype=sf.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for k_, v in pinned.items()
              if isinstance(v, torch.Tensor))
    d2h = o_host.numel() * o_host.element_size() + sf_host.numel() * 4
    sets = [dev, {key: (torch.empty_like(val) if isinstance(val, torch.Tensor) else val)
                  for key, val in dev.items()}]
    outs = [(o, sf), (torch.empty_like(o), torch.empty_like(sf))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_back = [torch.cuda.Event() for _ in range(2)]
    e2e_state = {"i": 0}

    def e2e_step():
        b = e2e_state["i"] & 1
        e2e_state["i"] += 1
        d, (ob, sfb) = sets[b], outs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[b])       # step i - 2 has read these inputs
            for key, val in pinned.items():
                if isinstance(val, torch.Tensor):
                    d[key].copy_(val, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_back[b])         # step i - 2's outputs are home
        ckda.ckda_fwd_chunked(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                              d["initial_state"], sfb, ob, d["cu_seqlens"], None,
                              chunk=w.chunk, stream=stream, workspace=ws)
        ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            o_host.copy_(ob, non_blocking=True)
            sf_host.copy_(sfb, non_blocking=True)
            ev_back[b].record(s_out)

    def e2e_loop(steps):
        for _ in range(steps):
            e2e_step()
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    for ev in ev_done + ev_back:
        ev.record(stream)
    e2e_loop(3)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    st_ev, en_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st_ev.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    e2e_loop(args.e2e_steps)
    en_ev.record(stream)
    en_ev.synchronize()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    if ckda.ckda_last_error() != ckda.CKDA_OK:
        raise RuntimeError("kernel reported an error")
    e2e_ms = st_ev.elapsed_time(en_ev) / args.e2e_steps
    if dist:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": T_total * world / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms,
           "pipeline": "copies in, forward and copies out on three streams, two buffer sets"}
    del sets[1], outs[1]

    # ---------------- the same workload through the fused input prologue
    ginp = make_gated_fwd_inputs(w)
    gdev = {key: (val.cuda() if isinstance(val, torch.Tensor) else val)
            for key, val in ginp.items()}
    gates = ckda.GateParams(**ckda.CKDA_GATES, k_eps=1e-6)

    def prefill_gated():
        ckda.ckda_fwd_chunked_gated(gdev["q"], gdev["k_raw"], gdev["v"], gdev["a_logit"],
                                    gdev["c_logit"], gdev["initial_state"], sf, o, gates,
                                    gdev["cu_seqlens"], None, chunk=w.chunk,
                                    stream=stream, workspace=ws)

    gms = time_loop(prefill_gated, args.steps, args.warmup, stream, barrier)
    gbytes = prefill_gated_bytes(ginp)
    gated = {"ms_per_step": gms, "tokens_per_s": T_total * world / (gms / 1e3),
             "roofline": {"bound": "hbm", "achieved": gbytes / (gms / 1e3) / 1e9,
                          "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": gbytes / (gms / 1e3) / 1e9 / pk["hbm_gbs"],
                          "traffic": None, "algorithmic_bytes_per_launch": gbytes},
             "inputs": "bf16 q, raw k, v, gate logits a; fp32 logits c; CKDA ranges",
             "gpu_launches": 3 * args.steps}
    del gdev

    # ---------------- backward pass of the same workload
    bg = make_bwd_grads(w, T_total, H, N)
    bdo, bdsf = bg["d_o"].cuda(), bg["d_final_state"].cuda()
    bout = [torch.empty_like(dev["q"]), torch.empty_like(dev["k"]), torch.empty_like(dev["v"]),
            torch.empty_like(dev["alpha"]), torch.empty_like(dev["beta"]),
            torch.empty((N, H, dk, dv), dtype=torch.float32, device="cuda")]
    bws = torch.empty(ckda.ckda_bwd_workspace_bytes(N, T_total, H, dk, dv, True,
                                                    args.bwd_impl == "chunked"),
                      dtype=torch.uint8, device="cuda")

    def bwd_step():
        ckda.ckda_bwd(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"],
                      dev["initial_state"], bdo, bdsf, *bout, dev["cu_seqlens"], None,
                      stream=stream, workspace=bws, chunked=args.bwd_impl == "chunked")

    bms = time_loop(bwd_step, args.bwd_steps, 3, stream, barrier)
    if ckda.ckda_last_error() != ckda.CKDA_OK:
        raise RuntimeError("kernel reported an error")
    bbytes = bwd_bytes(inp_cpu)
    backward = {"ms_per_step": bms, "tokens_per_s": T_total * world / (bms / 1e3),
                "steps": args.bwd_steps, "warmup": 3,
                "roofline": {"bound": "hbm", "achieved": bbytes / (bms / 1e3) / 1e9,
                             "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": bbytes / (bms / 1e3) / 1e9 / pk["hbm_gbs"],
                             "traffic": NCU_TRAFFIC["backward" if args.bwd_impl == "serial"
                                                    else "backward_chunked"],
                             "algorithmic_bytes_per_launch": bbytes},
                "kernel": ("token-serial adjoint on CUDA cores, one CTA per (sequence, head, "
                           "32-column tile), plus a tile reduction" if args.bwd_impl == "serial"
                           else "chunkwise (16-token chunk-WY reverse) on CUDA cores: prep and "
                                "gradients over all chunks, two scans per (sequence, head, "
                                "16-column tile) fed by asynchronous copies two chunks ahead"),
                "entry_point": "ckda_bwd_chunked" if args.bwd_impl == "chunked" else "ckda_bwd",
                "gpu_launches": (2 if args.bwd_impl == "serial" else 4) * args.bwd_steps}
    del bws, bout

    # ---------------- the complex-phase gate on the same shape (complex64)
    cin = {key: val.cuda() for key, val in
           make_complex_inputs(w, inp_cpu["cu_seqlens"], H).items()}
    co = torch.empty((T_total, H, dv), dtype=torch.complex64, device="cuda")
    csf = torch.empty((N, H, dk, dv), dtype=torch.complex64, device="cuda")

    cchunked = args.complex_impl == "chunked"
    cws = None
    if cchunked:
        cws = torch.empty(ckda.ckda_fwd_complex_chunked_workspace_bytes(N, T_total, H, dk, dv,
                                                                         True),
                          dtype=torch.uint8, device="cuda")

    def complex_step():
        ckda.ckda_fwd_complex(cin["q"], cin["k"], cin["v"], cin["alpha"], cin["theta"],
                              cin["beta"], cin["initial_state"], csf, co, cin["cu_seqlens"],
                              None, stream=stream, chunked=cchunked, workspace=cws)

    cms = time_loop(complex_step, args.complex_steps, 3, stream, barrier)
    if ckda.ckda_last_error() != ckda.CKDA_OK:
        raise RuntimeError("kernel reported an error")
    cbytes = complex_bytes(T_total, H, N, dk, dv)
    complex_gate = {"ms_per_step": cms, "tokens_per_s": T_total * world / (cms / 1e3),
                    "steps": args.complex_steps, "warmup": 3,
                    "roofline": {"bound": "hbm", "achieved": cbytes / (cms / 1e3) / 1e9,
                                 "peak": pk["hbm_gbs"], "unit": "GB/s",
                                 "frac": cbytes / (cms / 1e3) / 1e9 / pk["hbm_gbs"],
                                 "traffic": None, "algorithmic_bytes_per_launch": cbytes},
                    "kernel": ("chunked (16-token chunk-WY, complex) on CUDA cores, fp32: "
                               "a prep over all chunks and a state scan" if cchunked else
                               "token-serial complex recurrence on CUDA cores, fp32"),
                    "entry_point": ("ckda_fwd_complex_chunked" if cchunked
                                    else "ckda_fwd_complex"),
                    "gpu_launches": (2 if cchunked else 1) * args.complex_steps}
    del cws
    del cin, co, csf

    # ---------------- decode step
    wd = WORKLOADS[DECODE]
    state = make_decode_state(wd).cuda()
    toks = [{key: val.cuda() for key, val in make_decode_tokens(wd, s).items()}
            for s in range(4)]
    od = torch.empty((wd.B, wd.H, wd.d_v), dtype=toks[0]["q"].dtype, device="cuda")
    it = [0]

    def dstep():
        tk = toks[it[0] % len(toks)]
        it[0] += 1
        ckda.ckda_decode_step(tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"],
                              state, od, stream=stream)

    with ClockSampler(local) as dclk:
        dms = time_loop(dstep, args.decode_steps, args.warmup, stream, barrier)
    dbytes = decode_bytes(wd.B, wd.H, wd.d_k, wd.d_v, toks[0]["q"].dtype)
    dgbs = dbytes / (dms / 1e3) / 1e9
    decode = {"workload": DECODE, "ms_per_step": dms,
              "tokens_per_s": wd.B * world / (dms / 1e3),
              "token_heads_per_s": wd.B * wd.H * world / (dms / 1e3),
              "steps": args.decode_steps,
              "roofline": {"bound": "hbm", "achieved": dgbs, "peak": pk["hbm_gbs"],
                           "unit": "GB/s", "frac": dgbs / pk["hbm_gbs"],
                           "traffic": NCU_TRAFFIC["decode"],
                           "algorithmic_bytes_per_launch": dbytes},
              "gpu_launches": args.decode_steps, "clocks": dclk.summary()}

    extra = {}
    if not args.no_chunked_legs:
        extra = chunked_legs(args, w, inp_cpu, T_total, H, N, dk, dv, stream, pk, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_prefill(w, inp_cpu)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": PREFILL, "global_batch": world, "seq_len": T_total,
                   "heads": H, "d_k": dk, "d_v": dv, "chunk": w.chunk,
                   "io": "bf16 q/k/v/o, fp32 alpha/beta/state",
                   "l2": "inputs larger than L2 (%.0f MB per step)" % (nbytes / 1e6),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        # each forward call launches the slot-table, prep and scan kernels
        "gpu_launches": 3 * args.steps, "clocks": clk.summary(), "decode": decode,
        "prefill_fused_prologue": gated, "backward": backward, "complex_gate": complex_gate,
    }
    line.update(extra)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
