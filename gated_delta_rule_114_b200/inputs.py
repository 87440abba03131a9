"""Seeded synthetic inputs for the CKDA chunked forward and decode step.

This module is shared by the tests, the benchmark and the smoke check, and it
feeds both the CUDA library and the fp64 oracle. It holds none of the method's
arithmetic: it only draws random tensors with the shapes and distributions of
the five workloads below, L2-normalises q and k per token (the caller's job in
the recurrence's statement, "Semidirect Fourier Delta Attention" §3 eq. (18)
without its epsilon), and casts to the I/O dtype.

Draw recipe (CPU ``torch.Generator``, fp32, fixed order):
  q, k, v, alpha-normal, alpha-mask, beta-normal, initial state.
For the varlen workload the sequence lengths come first, from their own
generator (seed + 7919), because the token count depends on them.
q and k are normalised in fp32 and then cast; alpha, beta and states stay fp32.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    H: int
    d_k: int
    d_v: int
    dtype: str              # "f32" or "bf16": dtype of q, k, v, o
    chunk: int              # chunk length the forward is run with
    B: int = 1              # equal-length sequences (ignored when varlen)
    T: int = 0              # per-sequence length (equal-length workloads)
    varlen_n: int = 0       # >0: number of packed sequences
    varlen_lo: int = 0
    varlen_hi: int = 0
    alpha_kind: str = "tanh1.5"
    beta_kind: str = "2sig1"
    init_state: bool = False
    decode: bool = False


# The five workloads of the CKDA forward / decode path.
WORKLOADS = {
    # tiny fp32 check of the chunk algebra
    "tiny_T64_d16_f32": Workload(
        name="tiny_T64_d16_f32", seed=1001, B=1, H=1, T=64, d_k=16, d_v=16,
        dtype="f32", chunk=16, alpha_kind="tanh1.5", beta_kind="2sig1"),
    # KDA ranges: alpha in (0,1), beta in (0,1)
    "kda_B4_H16_T2048_d128": Workload(
        name="kda_B4_H16_T2048_d128", seed=1002, B=4, H=16, T=2048, d_k=128,
        d_v=128, dtype="bf16", chunk=64, alpha_kind="kda", beta_kind="sig1"),
    # CKDA ranges, long prefill (the headline forward)
    "ckda_B1_H32_T8192_d128": Workload(
        name="ckda_B1_H32_T8192_d128", seed=1003, B=1, H=32, T=8192,
        d_k=128, d_v=128, dtype="bf16", chunk=64, alpha_kind="ckda",
        beta_kind="2sig1.5", init_state=True),
    # CKDA ranges, 32 packed sequences of U[128, 4096] tokens
    "ckda_varlen_N32_H32_d128": Workload(
        name="ckda_varlen_N32_H32_d128", seed=1004, H=32, d_k=128, d_v=128,
        dtype="bf16", chunk=64, varlen_n=32, varlen_lo=128, varlen_hi=4096,
        alpha_kind="ckda", beta_kind="2sig1.5", init_state=True),
    # decode: 256 sequences x 32 heads, one token per step
    "decode_N256_H32_d128": Workload(
        name="decode_N256_H32_d128", seed=1005, B=256, H=32, T=1, d_k=128,
        d_v=128, dtype="bf16", chunk=1, alpha_kind="tanh2", beta_kind="2sig1",
        init_state=True, decode=True),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _alpha(kind: str, shape, g: torch.Generator) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    u = torch.rand(shape, generator=g, dtype=torch.float32)
    if kind == "tanh1.5":
        return torch.tanh(1.5 * x)
    if kind == "tanh2":
        return torch.tanh(2.0 * x)
    if kind == "kda":  # exp(-softplus(x)) in (0, 1)
        return torch.exp(-torch.nn.functional.softplus(x))
    if kind == "ckda":  # tanh(N(0,2)); 5% exactly +-1 (fair sign), 1% exactly 0
        a = torch.tanh(2.0 * x)
        a = torch.where(u < 0.025, torch.ones_like(a), a)
        a = torch.where((u >= 0.025) & (u < 0.05), -torch.ones_like(a), a)
        a = torch.where((u >= 0.05) & (u < 0.06), torch.zeros_like(a), a)
        return a
    if kind == "slow":  # long memory: |alpha| = 1 - 0.01 |N(0,1)|, 10% negative
        a = 1.0 - 0.01 * x.abs()
        return torch.where(u < 0.1, -a, a)
    raise ValueError(kind)


def _beta(kind: str, shape, g: torch.Generator) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if kind == "2sig1":
        return 2.0 * torch.sigmoid(x)
    if kind == "sig1":
        return torch.sigmoid(x)
    if kind == "2sig1.5":
        return 2.0 * torch.sigmoid(1.5 * x)
    raise ValueError(kind)


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def seqlens(w: Workload) -> torch.Tensor:
    """int32 [N+1] cumulative sequence lengths for a workload."""
    if w.varlen_n > 0:
        g = _gen(w.seed + 7919)
        lens = torch.randint(w.varlen_lo, w.varlen_hi + 1, (w.varlen_n,),
                             generator=g, dtype=torch.int64)
    else:
        lens = torch.full((w.B,), w.T, dtype=torch.int64)
    cu = torch.zeros(lens.numel() + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    return cu.to(torch.int32)


def make_fwd_inputs(w: Workload, cu_seqlens: torch.Tensor | None = None,
                    H: int | None = None) -> dict:
    """CPU tensors for one forward call of workload ``w``.

    Returns q, k, v (I/O dtype), alpha, beta, initial_state (fp32 or None),
    cu_seqlens (int32 [N+1]). ``cu_seqlens``/``H`` override the workload's
    lengths/heads (used for reduced-size parity cases with the same recipe).
    """
    g = _gen(w.seed)
    cu = seqlens(w) if cu_seqlens is None else cu_seqlens.to(torch.int32)
    H = w.H if H is None else H
    N = cu.numel() - 1
    T = int(cu[-1])
    dt = TORCH_DTYPE[w.dtype]
    q = _unit(torch.randn(T, H, w.d_k, generator=g, dtype=torch.float32))
    k = _unit(torch.randn(T, H, w.d_k, generator=g, dtype=torch.float32))
    v = torch.randn(T, H, w.d_v, generator=g, dtype=torch.float32)
    alpha = _alpha(w.alpha_kind, (T, H, w.d_k), g)
    beta = _beta(w.beta_kind, (T, H), g)
    s0 = None
    if w.init_state:
        s0 = 0.1 * torch.randn(N, H, w.d_k, w.d_v, generator=g,
                               dtype=torch.float32)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), alpha=alpha.contiguous(),
                beta=beta.contiguous(), initial_state=s0, cu_seqlens=cu)


def make_decode_state(w: Workload, N: int | None = None,
                      H: int | None = None) -> torch.Tensor:
    """fp32 [N, H, d_k, d_v] initial decode state, N(0, 0.1)."""
    g = _gen(w.seed)
    N = w.B if N is None else N
    H = w.H if H is None else H
    return 0.1 * torch.randn(N, H, w.d_k, w.d_v, generator=g,
                             dtype=torch.float32)


def make_decode_tokens(w: Workload, step: int, N: int | None = None,
                       H: int | None = None) -> dict:
    """Fresh seeded tokens for decode step ``step`` (seed = seed*100003+step)."""
    g = _gen(w.seed * 100003 + int(step))
    N = w.B if N is None else N
    H = w.H if H is None else H
    dt = TORCH_DTYPE[w.dtype]
    q = _unit(torch.randn(N, H, w.d_k, generator=g, dtype=torch.float32))
    k = _unit(torch.randn(N, H, w.d_k, generator=g, dtype=torch.float32))
    v = torch.randn(N, H, w.d_v, generator=g, dtype=torch.float32)
    alpha = _alpha(w.alpha_kind, (N, H, w.d_k), g)
    beta = _beta(w.beta_kind, (N, H), g)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), alpha=alpha.contiguous(),
                beta=beta.contiguous())


def token_heads(w: Workload) -> int:
    cu = seqlens(w)
    return int(cu[-1]) * w.H


def _gate_logits(shape, g: torch.Generator) -> torch.Tensor:
    """Gate logits a ~ N(0, 2); 1% exactly 0 and 5% +-30 (fair sign), which
    the fused prologue with the CKDA ranges maps to alpha = 0 and, in fp32,
    alpha = +-1 exactly."""
    x = 2.0 * torch.randn(shape, generator=g, dtype=torch.float32)
    u = torch.rand(shape, generator=g, dtype=torch.float32)
    x = torch.where(u < 0.025, torch.full_like(x, 30.0), x)
    x = torch.where((u >= 0.025) & (u < 0.05), torch.full_like(x, -30.0), x)
    return torch.where((u >= 0.05) & (u < 0.06), torch.zeros_like(x), x)


def _raw_keys(shape, g: torch.Generator) -> torch.Tensor:
    """Unnormalised keys: N(0, 1) rows scaled by U(0.2, 3) per row."""
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    s = 0.2 + 2.8 * torch.rand(shape[:-1] + (1,), generator=g, dtype=torch.float32)
    return x * s


def make_gated_fwd_inputs(w: Workload, cu_seqlens: torch.Tensor | None = None,
                          H: int | None = None) -> dict:
    """CPU tensors for one forward with the fused input prologue: q (unit
    rows), k_raw, v, a_logit (I/O dtype), c_logit ~ N(0, 1.5) (fp32),
    initial_state, cu_seqlens; shapes as make_fwd_inputs."""
    g = _gen(w.seed + 31337)
    cu = seqlens(w) if cu_seqlens is None else cu_seqlens.to(torch.int32)
    H = w.H if H is None else H
    N = cu.numel() - 1
    T = int(cu[-1])
    dt = TORCH_DTYPE[w.dtype]
    q = _unit(torch.randn(T, H, w.d_k, generator=g, dtype=torch.float32))
    k = _raw_keys((T, H, w.d_k), g)
    v = torch.randn(T, H, w.d_v, generator=g, dtype=torch.float32)
    a = _gate_logits((T, H, w.d_k), g)
    c = 1.5 * torch.randn(T, H, generator=g, dtype=torch.float32)
    s0 = None
    if w.init_state:
        s0 = 0.1 * torch.randn(N, H, w.d_k, w.d_v, generator=g, dtype=torch.float32)
    return dict(q=q.to(dt), k_raw=k.to(dt), v=v.to(dt), a_logit=a.to(dt).contiguous(),
                c_logit=c.contiguous(), initial_state=s0, cu_seqlens=cu)


def make_gated_decode_tokens(w: Workload, step: int, N: int | None = None,
                             H: int | None = None) -> dict:
    """Fresh seeded tokens with logits for a gated decode step."""
    g = _gen(w.seed * 100003 + 7777 + int(step))
    N = w.B if N is None else N
    H = w.H if H is None else H
    dt = TORCH_DTYPE[w.dtype]
    q = _unit(torch.randn(N, H, w.d_k, generator=g, dtype=torch.float32))
    k = _raw_keys((N, H, w.d_k), g)
    v = torch.randn(N, H, w.d_v, generator=g, dtype=torch.float32)
    a = _gate_logits((N, H, w.d_k), g)
    c = 1.5 * torch.randn(N, H, generator=g, dtype=torch.float32)
    return dict(q=q.to(dt), k_raw=k.to(dt), v=v.to(dt), a_logit=a.to(dt).contiguous(),
                c_logit=c.contiguous())


def make_bwd_grads(w: Workload, T_total: int, H: int, N: int, seed_offset: int = 0) -> dict:
    """Seeded upstream gradients for a backward pass: d_o ~ N(0, 1)
    [T_total, H, d_v] in the I/O dtype and d_final_state ~ N(0, 1)
    [N, H, d_k, d_v] fp32."""
    g = _gen(w.seed + 4242 + seed_offset)
    d_o = torch.randn(T_total, H, w.d_v, generator=g, dtype=torch.float32)
    dsf = torch.randn(N, H, w.d_k, w.d_v, generator=g, dtype=torch.float32)
    return dict(d_o=d_o.to(TORCH_DTYPE[w.dtype]), d_final_state=dsf)


def make_complex_inputs(w: Workload, cu_seqlens: torch.Tensor, H: int, theta_max: float = 1.5,
                        ranges: str = "sfda", seed_offset: int = 0) -> dict:
    """Seeded inputs for the complex-phase gate: q, k (unit rows), v complex64
    with N(0, 1) real and imaginary parts; theta = theta_max tanh(N(0, 1));
    ranges "sfda": alpha = sigmoid(N(0, 1)) in (0, 1), beta = sigmoid(N(0, 1));
    "ckda": alpha = tanh(N(0, 2)) in (-1, 1), beta = 2 sigmoid(N(0, 1.5));
    initial state N(0, 0.1) complex64."""
    g = _gen(w.seed + 9090 + seed_offset)
    cu = cu_seqlens.to(torch.int32)
    N, T = cu.numel() - 1, int(cu[-1])

    def cn(*shape):
        re = torch.randn(*shape, generator=g, dtype=torch.float32)
        im = torch.randn(*shape, generator=g, dtype=torch.float32)
        return torch.complex(re, im)

    q = cn(T, H, w.d_k)
    k = cn(T, H, w.d_k)
    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    v = cn(T, H, w.d_v)
    theta = theta_max * torch.tanh(torch.randn(T, H, w.d_k, generator=g))
    if ranges == "ckda":
        alpha = torch.tanh(2.0 * torch.randn(T, H, w.d_k, generator=g))
        beta = 2.0 * torch.sigmoid(1.5 * torch.randn(T, H, generator=g))
    else:
        alpha = torch.sigmoid(torch.randn(T, H, w.d_k, generator=g))
        beta = torch.sigmoid(torch.randn(T, H, generator=g))
    s0 = 0.1 * cn(N, H, w.d_k, w.d_v)
    return dict(q=q, k=k, v=v, alpha=alpha.contiguous(), theta=theta.contiguous(),
                beta=beta.contiguous(), initial_state=s0, cu_seqlens=cu)
