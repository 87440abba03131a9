"""The no-allocation forward against the regular one (GPU).

ckda_fwd_chunked_noalloc serves callers that cannot give the library device
memory (a plain C caller with no allocator, or a loop that must not call
cudaMalloc while it runs): its scratch is a fixed array inside the library.
These tests call it through the C ABI and compare with ckda_fwd_chunked run
on a workspace from torch, on two calls in a row with different inputs (the
shared array keeps the first call's contents when the second one starts).
This file is collected after the other test files and its tests are marked
``last`` too, so they run after every other test (tests/conftest.py keeps the
collected order inside the ``last`` group), and a run stopping at the first
failure has already run the rest. Both entry points run the same deterministic
kernels, so their results must agree bit for bit.
"""
import dataclasses

import pytest
import torch

from gated_delta_rule_114_b200 import ckda
from gated_delta_rule_114_b200.inputs import WORKLOADS, make_fwd_inputs
from parity_util import to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.last]


def _inputs(seed, lens, H):
    w = dataclasses.replace(WORKLOADS["ckda_B1_H32_T8192_d128"], seed=seed)
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    return to_dev(make_fwd_inputs(w, cu_seqlens=cu, H=H)), cu


def _regular(d, cu):
    o = torch.empty_like(d["v"])
    sf = torch.empty_like(d["initial_state"])
    ckda.ckda_fwd_chunked(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                          d["initial_state"], sf, o, d["cu_seqlens"], cu)
    return o, sf


def _noalloc(d, cu):
    o = torch.empty_like(d["v"])
    sf = torch.empty_like(d["initial_state"])
    ckda.ckda_fwd_chunked_noalloc(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                  d["initial_state"], sf, o, d["cu_seqlens"], cu)
    return o, sf


def test_noalloc_matches_regular_on_two_calls(cuda_lib):
    for seed, lens, H in ((71, [100, 37, 64], 4), (72, [130, 1, 90], 3)):
        d, cu = _inputs(seed, lens, H)
        need = ckda.ckda_fwd_workspace_bytes(len(lens), sum(lens), H, 128, 128,
                                             varlen=True)
        assert 0 < need <= ckda.NOALLOC_SCRATCH_BYTES
        o_ref, sf_ref = _regular(d, cu)
        o, sf = _noalloc(d, cu)
        torch.cuda.synchronize()
        assert ckda.ckda_last_error() == ckda.CKDA_OK
        assert torch.equal(o, o_ref) and torch.equal(sf, sf_ref)


def _largest_fitting_T(H):
    """Largest single-sequence length whose scratch fits the fixed array."""
    T = 64
    while ckda.ckda_fwd_workspace_bytes(1, T + 1, H, 128, 128) <= ckda.NOALLOC_SCRATCH_BYTES:
        T += 1
    return T


def test_noalloc_at_its_size_limit(cuda_lib):
    """The largest call the array holds (32 heads, one sequence) runs and
    agrees bit for bit with the regular entry point."""
    H = 32
    T = _largest_fitting_T(H)
    d, cu = _inputs(73, [T], H)
    o_ref, sf_ref = _regular(d, cu)
    o, sf = _noalloc(d, cu)
    torch.cuda.synchronize()
    assert ckda.ckda_last_error() == ckda.CKDA_OK
    assert torch.equal(o, o_ref) and torch.equal(sf, sf_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    """One token more than the limit above needs more scratch than the array
    has: the call is refused and launches nothing."""
    H = 32
    T = _largest_fitting_T(H) + 1
    assert ckda.ckda_fwd_workspace_bytes(1, T, H, 128, 128) > ckda.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
    a = torch.ones(T, H, 128, device="cuda")
    b = torch.zeros(T, H, device="cuda")
    o = torch.full_like(q, 7.0)
    with pytest.raises(ckda.CkdaError) as e:
        ckda.ckda_fwd_chunked_noalloc(q, q, q, a, b, None, None, o, N=1, T=T)
    assert e.value.status == ckda.CKDA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((o == 7.0).all())
