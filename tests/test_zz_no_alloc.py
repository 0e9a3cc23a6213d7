"""kda_forward_noalloc, the entry point for callers that cannot allocate device
memory (engines that pre-plan all device memory in their own pools, hosts that
hand over raw device pointers without an allocator): called through the C ABI,
it must give the same results as kda_forward with a caller-provided workspace,
on two calls in a row with different batches (the second one finds the
previous call's schedule in the shared scratch array), and refuse packed
batches larger than that array.

This file is named to be collected last, so a run that stops at its first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from kda_testutil import TOL, case, rel
from linear_attention_recurrence_11_b200.inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_c(K, inp, o, ST, chunk=64):
    """The raw C-ABI call (no Python-side checks in between)."""
    cu = inp.get("cu_seqlens")
    B, T, H, dk = inp["k"].shape
    dv = inp["v"].shape[-1]
    nseq = 0 if cu is None else cu.numel() - 1
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    rc = K._lib.kda_forward_noalloc(
        _ptr(inp["q"]), _ptr(inp["k"]), _ptr(inp["v"]), _ptr(inp["g"]), _ptr(inp["beta"]),
        _ptr(inp.get("S0")), _ptr(o), _ptr(ST), B, T, H, dk, dv, chunk, K.DTYPES[inp["k"].dtype],
        _ptr(cu), nseq, _ptr(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, int(status[0])


@pytest.mark.parametrize("dtype,dk,chunk", [("bf16", 128, 64), ("f32", 64, 32)])
def test_noalloc_matches_forward_two_calls(K, dtype, dk, chunk):
    """Two calls in a row with different packed batches: the second has more
    sequences, in another length order, so its longest-first schedule differs
    from the one the first call leaves in the shared array (every stale entry is
    still a valid sequence index of the second batch, so a call that read the
    array without writing it would run some sequences twice and others never,
    and its NaN-filled outputs would show it). Each call is compared with
    kda_forward (caller-provided workspace) on the same inputs."""
    batches = [[7, 130, 0, 200, 1, 65, 33],
               [300, 1, 90, 0, 12, 65, 200, 7, 0, 130, 33, 64]]
    for call, lens in enumerate(batches):
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        inp = case(1, int(cu[-1]), 3, dk, dk, dtype, seed=77 + call, s0_std=0.1, num_states=len(lens))
        inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
        o_ref, S_ref = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"],
                                     chunk=chunk, cu_seqlens=inp["cu_seqlens"])
        torch.cuda.synchronize()
        o = torch.full_like(o_ref, float("nan"))
        ST = torch.full_like(S_ref, float("nan"))
        rc, status = _noalloc_c(K, inp, o, ST, chunk)
        assert rc == 0 and status == 0, (call, rc, status)
        assert torch.isfinite(o).all() and torch.isfinite(ST).all(), call
        assert rel(to_f64(o), to_f64(o_ref)) < TOL[dtype], call
        assert rel(to_f64(ST), to_f64(S_ref)) < TOL[dtype], call


def test_noalloc_dense_batch_and_scratch_limit(K):
    inp = case(2, 150, 2, 128, 128, "bf16", seed=78, s0_std=0.1)
    o_ref, S_ref = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64)
    o, ST = torch.empty_like(o_ref), torch.empty_like(S_ref)
    K.kda_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], o, ST, chunk=64)
    torch.cuda.synchronize()
    assert rel(to_f64(o), to_f64(o_ref)) < TOL["bf16"] and rel(to_f64(ST), to_f64(S_ref)) < TOL["bf16"]
    # more packed sequences than the fixed scratch holds: refused, nothing launched
    n = 2049
    cu = torch.arange(n + 1, dtype=torch.int32, device="cuda")
    small = case(1, n, 1, 128, 128, "bf16", seed=79)
    small["cu_seqlens"] = cu
    o2 = torch.empty(1, n, 1, 128, dtype=torch.bfloat16, device="cuda")
    rc, _ = _noalloc_c(K, small, o2, None)
    assert rc == K.KDA_ERR_SCRATCH_LIMIT
    assert "scratch" in K.kda_status_string(rc)
