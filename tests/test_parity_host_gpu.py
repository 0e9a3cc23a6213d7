"""GPU tests of the prefill from host memory (kda_forward_host): the pieces,
copied up, run from the carried state and copied down, give the same o and
S_T as one device-resident kda_forward_ex call over the whole sequence (bit
for bit, pieces being whole chunks), and meet the oracle's bars."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_11_b200.inputs import WORKLOADS, to_f64, workload_inputs

from kda_testutil import TOL, case, compare_units, oracle_forward, rel

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "g", "beta")


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def to_host(inp, pinned=True):
    out = {}
    for n in NAMES + ("S0",):
        t = inp.get(n)
        if t is not None:
            t = t.cpu()
            out[n] = t.pin_memory() if pinned else t
    return out


def run_host(K, hinp, chunk, piece_len, path="auto", stream=None):
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, S_T = K.kda_forward_host(*(hinp[n] for n in NAMES), hinp.get("S0"), chunk=chunk, piece_len=piece_len,
                                path=path, dev_status=status, stream=stream)
    (stream or torch.cuda.current_stream()).synchronize()
    assert int(status[0]) == 0
    return o, S_T


def run_device(K, inp, chunk, path="auto"):
    o, S_T = K.kda_forward(*(inp[n] for n in NAMES), inp.get("S0"), chunk=chunk, path=path)
    torch.cuda.synchronize()
    return o.cpu(), S_T.cpu()


@pytest.mark.parametrize("B,T,piece_len,s0", [
    (1, 700, 192, 0.1),   # ragged last piece and chunk
    (2, 512, 128, 0.0),   # B > 1: strided copies; pieces end on the sequence end
    (2, 300, 0, 0.5),     # default piece length
    (1, 64, 640, 0.1),    # one piece, shorter than piece_len
])
def test_bf16_pieces_equal_one_device_call(K, B, T, piece_len, s0):
    inp = case(B, T, 3, 128, 128, "bf16", seed=T + piece_len, s0_std=s0)
    o, S_T = run_host(K, to_host(inp), 64, piece_len)
    o_d, S_d = run_device(K, inp, 64)
    assert torch.equal(o, o_d) and torch.equal(S_T, S_d)


@pytest.mark.parametrize("dtype,dk,dv,chunk,T,piece_len", [
    ("f32", 64, 32, 32, 301, 96), ("f32", 128, 128, 64, 256, 64), ("bf16", 64, 128, 16, 200, 48),
])
def test_simt_shapes_equal_one_device_call(K, dtype, dk, dv, chunk, T, piece_len):
    inp = case(2, T, 2, dk, dv, dtype, seed=dk + dv + T, s0_std=0.1)
    o, S_T = run_host(K, to_host(inp), chunk, piece_len)
    o_d, S_d = run_device(K, inp, chunk)
    assert torch.equal(o, o_d) and torch.equal(S_T, S_d)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_oracle_parity_through_host_buffers(K, oracle_mod, dtype):
    inp = case(2, 333, 2, 128, 64 if dtype == "f32" else 128, dtype, seed=31, s0_std=0.1)
    o, S_T = run_host(K, to_host(inp), 64 if dtype == "bf16" else 32, 128 if dtype == "bf16" else 64)
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    units = [(b, h) for b in range(2) for h in range(2)]
    e_o, e_s = compare_units(o, S_T, o_ref, S_ref, units, tol=TOL[dtype])
    assert e_o < TOL[dtype] and e_s < TOL[dtype], (e_o, e_s)


def test_no_initial_state_and_pageable_memory(K):
    inp = case(1, 400, 2, 128, 128, "bf16", seed=33)
    inp.pop("S0", None)
    o, S_T = run_host(K, to_host(inp, pinned=False), 64, 128)
    o_d, S_d = run_device(K, inp, 64)
    assert torch.equal(o, o_d) and torch.equal(S_T, S_d)


def test_empty_sequence_returns_the_initial_state(K):
    inp = case(2, 64, 2, 128, 128, "bf16", seed=35, s0_std=0.3)
    h = to_host(inp)
    h = {n: (t[:, :0].contiguous() if n in NAMES else t) for n, t in h.items()}
    o, S_T = run_host(K, h, 64, 64)
    assert o.shape[1] == 0 and torch.equal(S_T, h["S0"])


def test_side_stream_and_back_to_back_calls(K):
    """Two calls in a row on a non-default stream with one workspace: the
    stream order makes the second wait for the first's downloads."""
    a = case(1, 640, 2, 128, 128, "bf16", seed=37, s0_std=0.1)
    b = case(1, 640, 2, 128, 128, "bf16", seed=38, s0_std=0.1)
    s = torch.cuda.Stream()
    ws = torch.empty(K.kda_forward_host_workspace_size(1, 640, 2, 128, 128, 64, torch.bfloat16, 128),
                     dtype=torch.uint8, device="cuda")
    ha, hb = to_host(a), to_host(b)
    oa, Sa = K.kda_forward_host(*(ha[n] for n in NAMES), ha["S0"], piece_len=128, workspace=ws, stream=s)
    ob, Sb = K.kda_forward_host(*(hb[n] for n in NAMES), hb["S0"], piece_len=128, workspace=ws, stream=s)
    s.synchronize()
    for (o, S), inp in (((oa, Sa), a), ((ob, Sb), b)):
        o_d, S_d = run_device(K, inp, 64)
        assert torch.equal(o, o_d) and torch.equal(S, S_d)


def test_benchmark_workload_sampled(K, oracle_mod):
    """The 96-head, 8192-token workload in the configuration the end-to-end
    benchmark times (pieces of 1024 tokens): equal to the device call, and two
    heads against the oracle."""
    w = WORKLOADS["prefill_h96_T8192_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    o, S_T = run_host(K, to_host(inp), w.chunk, 1024)
    o_d, S_d = run_device(K, inp, w.chunk)
    assert torch.equal(o, o_d) and torch.equal(S_T, S_d)
    units = [(0, 0), (0, 57)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp, units=units)
    e_o, e_s = compare_units(o, S_T, o_ref, S_ref, units, tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)


def packed_host_case(lens, H, dk, dv, dtype, seed, s0_std):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    inp = case(1, int(cu[-1]), H, dk, dv, dtype, seed=seed, s0_std=s0_std, num_states=len(lens))
    inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
    return inp, cu


@pytest.mark.parametrize("lens,piece_len,s0", [
    ([300, 0, 700, 64, 5, 1000], 256, 0.1),   # cuts inside sequences, snapped to their chunk grids
    ([100, 200, 0], 128, 0.0),               # an empty sequence at the end; no S0
    ([64] * 10 + [0, 129], 192, 0.1),         # many short sequences per piece
    ([2048], 0, 0.1),                         # one sequence, default piece length
])
def test_packed_host_pieces(K, oracle_mod, lens, piece_len, s0):
    """Packed batches from host memory (kda_forward_host with cu_seqlens): pieces of the
    flat token axis, every cut on the chunk grid of the sequence it falls in, each a packed
    launch over the states of the sequences it touches. Against one device call over the
    whole batch (equal up to rounding: a piece may run another tensor-core form) and the
    oracle, every unit gated; empty sequences keep S0 bit for bit."""
    H = 2
    inp, cu = packed_host_case(lens, H, 128, 128, "bf16", seed=len(lens) + int(cu_sum(lens)), s0_std=s0)
    h = to_host(inp)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, S_T = K.kda_forward_host(*(h[n] for n in NAMES), h.get("S0"), chunk=64, piece_len=piece_len,
                                cu_seqlens=torch.tensor(cu), dev_status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    o_d, S_d = K.kda_forward(*(inp[n] for n in NAMES), inp.get("S0"), chunk=64, cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    o_d, S_d = o_d.cpu(), S_d.cpu()
    units = [(n, hh) for n in range(len(lens)) for hh in range(H)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    compare_units(o, S_T, o_ref, S_ref, units, [int(x) for x in cu], tol=TOL["bf16"], label="packed host")
    assert rel(to_f64(o), to_f64(o_d)) < 1e-2 and rel(to_f64(S_T), to_f64(S_d)) < 1e-2
    for n, L in enumerate(lens):
        if L == 0:
            want = inp["S0"][n].cpu() if inp.get("S0") is not None else torch.zeros_like(S_T[n])
            assert torch.equal(S_T[n], want)


def test_packed_host_fp32_simt(K, oracle_mod):
    lens = [90, 33, 0, 160]
    H = 2
    inp, cu = packed_host_case(lens, H, 64, 32, "f32", seed=5, s0_std=0.1)
    h = to_host(inp)
    o, S_T = K.kda_forward_host(*(h[n] for n in NAMES), h.get("S0"), chunk=32, piece_len=64,
                                cu_seqlens=torch.tensor(cu))
    torch.cuda.synchronize()
    units = [(n, hh) for n in range(len(lens)) for hh in range(H)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    compare_units(o, S_T, o_ref, S_ref, units, [int(x) for x in cu], tol=TOL["f32"], label="packed host f32")


def cu_sum(lens):
    return sum(lens)
