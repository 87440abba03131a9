"""Shared helpers of the GPU parity tests: tolerances and marshalling.

Tolerances (stated once, used by every parity test):
  * fp32 I/O check mode: max|x - x_ref| <= 1e-5 * rms(x_ref), for o and for
    the final state.
  * bf16 I/O with fp32 state and accumulation: the kernel's value before its
    final bf16 store must satisfy max|x - x_ref| <= 1e-2 * rms(x_ref). The
    store rounds to the nearest bf16, which moves a value by at most half a
    unit in the last place, i.e. at most 2^-8 |x|; the check therefore allows
    |o - o_ref| <= 1e-2 * rms(o_ref) + 2^-8 |o_ref| element by element. The
    final state is stored in fp32 and gets the plain 1e-2 * rms bound.
The oracle's reference values are computed in fp64 from the very values the
kernel sees (bf16-rounded q, k, v upcast exactly).

Every check records its literal max|x - x_ref| / rms(x_ref) in RECORDED;
the test session prints them at its end (tests/conftest.py), so that the
margin of each comparison, and for bf16 outputs how much of the store
allowance it used, shows in the output of a passing run.
"""
from __future__ import annotations

import os

import numpy as np
import torch

FP32_REL = 1e-5
BF16_REL = 1e-2
BF16_STORE = 2.0 ** -8

# (test id, what, literal max|x - x_ref| / rms(x_ref), bound factor, store ulp)
RECORDED: list = []


def rms(x: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(x)))) if x.size else 0.0


def as_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def check_close(x, x_ref, rel: float, store_ulp: float = 0.0, what: str = ""):
    """Assert max(|x - x_ref| - store_ulp*|x_ref|) <= rel * rms(x_ref)."""
    x = as_f64(x)
    x_ref = as_f64(x_ref)
    test_id = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    assert x.shape == x_ref.shape, (what, x.shape, x_ref.shape)
    assert np.all(np.isfinite(x)), what + ": non-finite output"
    if x.size == 0:
        RECORDED.append((test_id, what, 0.0, rel, store_ulp))
        return 0.0
    r = rms(x_ref)
    err = np.abs(x - x_ref)
    excess = err - store_ulp * np.abs(x_ref)
    worst = float(excess.max())
    bound = rel * r
    RECORDED.append((test_id, what, float(err.max()) / max(r, 1e-300), rel, store_ulp))
    assert worst <= bound, ("%s: max excess %.3e > %.3e (rel %.1e of rms %.3e); "
                            "literal max|x-x_ref|/rms = %.3e"
                            % (what, worst, bound, rel, r, float(err.max()) / max(r, 1e-300)))
    return float(err.max()) / max(r, 1e-300)


def check_bf16_out(o, o_ref, what="o"):
    return check_close(o, o_ref, BF16_REL, BF16_STORE, what)


def check_fp32(x, x_ref, what=""):
    return check_close(x, x_ref, FP32_REL, 0.0, what)


def to_dev(inp: dict, device="cuda") -> dict:
    out = {}
    for key, val in inp.items():
        out[key] = val.to(device).contiguous() if isinstance(val, torch.Tensor) else val
    return out


def poison(inp: dict, a: int, b: int, keys) -> None:
    """Overwrite tokens a .. b-1 of the inputs named by `keys` with NaN (the
    first few with +inf), in place."""
    for key in keys:
        x = inp[key].clone()
        x[a:b] = float("nan")
        x[a:min(b, a + 5)] = float("inf")
        inp[key] = x


def select_seqs(inp: dict, keep, keys):
    """The packed inputs of sequences `keep` only (their token rows, initial
    states and cu_seqlens), and the token rows they came from."""
    cu = inp["cu_seqlens"].tolist()
    idx = torch.cat([torch.arange(cu[n], cu[n + 1]) for n in keep])
    sub = {key: inp[key][idx] for key in keys}
    lens = [cu[n + 1] - cu[n] for n in keep]
    sub["cu_seqlens"] = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    s0 = inp.get("initial_state")
    sub["initial_state"] = None if s0 is None else s0[list(keep)]
    return sub, idx
