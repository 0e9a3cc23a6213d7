"""GPU parity of the segment-parallel prefill (segment pairs, scan, replay)
against the fp64 oracle, through the C ABI. Same bars as the plain prefill:
normwise 1e-4 for fp32 inputs, 1e-2 for bf16 inputs."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_11_b200.inputs import WORKLOADS, to_f64, workload_inputs

from kda_testutil import TOL, case, compare_units, oracle_forward, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def run_seg(K, inp, chunk, seg_len, path="auto"):
    status = torch.zeros(4, dtype=torch.int32, device=inp["k"].device)
    o, ST = K.kda_forward_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"),
                                    seg_len=seg_len, chunk=chunk, path=path, dev_status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0, f"device status {int(status[0])}"
    return o, ST


def check(K, oracle_mod, inp, chunk, seg_len, dtype, path):
    o, ST = run_seg(K, inp, chunk, seg_len, path)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    B, _, H, _ = inp["k"].shape
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, [(b, h) for b in range(B) for h in range(H)], tol=TOL[dtype])
    assert e_o < TOL[dtype] and e_s < TOL[dtype], (e_o, e_s)
    return o, ST


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("B,T,seg_len,s0", [(1, 1000, 256, 0.1), (2, 700, 128, 0.0), (1, 4 * 64, 64, 0.5)])
def test_bf16_segments(K, oracle_mod, path, B, T, seg_len, s0):
    """Several segments, a ragged last segment and chunk, with and without S0."""
    inp = case(B, T, 2, 128, 128, "bf16", seed=T + seg_len, s0_std=s0)
    check(K, oracle_mod, inp, 64, seg_len, "bf16", path)


@pytest.mark.parametrize("dtype,dk,dv,chunk,T,seg_len", [
    ("f32", 32, 32, 16, 256, 64), ("f32", 64, 32, 32, 301, 96), ("bf16", 64, 128, 16, 200, 48),
    ("f32", 128, 64, 64, 390, 128),
])
def test_simt_shapes(K, oracle_mod, dtype, dk, dv, chunk, T, seg_len):
    """The SIMT kernel serves both passes: fp32 at the 1e-4 bar, dk != dv (the
    transition pass runs with dv = dk)."""
    inp = case(2, T, 2, dk, dv, dtype, seed=dk * 3 + dv + T, s0_std=0.1)
    check(K, oracle_mod, inp, chunk, seg_len, dtype, "auto")


def test_g_min_segments(K, oracle_mod):
    """Decays pinned at g_min = -5 over whole segments: the transitions M_p are
    far from the identity and the scan carries almost nothing across."""
    inp = case(1, 512, 2, 128, 128, "bf16", seed=21, s0_std=0.1)
    inp["g"][:, :, :, ::2] = -5.0
    inp["g"][:, 128:320] = -5.0
    check(K, oracle_mod, inp, 64, 128, "bf16", "auto")


def test_one_segment_is_the_plain_prefill(K):
    """seg_len >= T: one segment, the call is kda_forward_ex (bit-identical)."""
    inp = case(2, 300, 2, 128, 128, "bf16", seed=23, s0_std=0.1)
    o1, S1 = run_seg(K, inp, 64, 320)
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_segments_agree_with_plain_prefill(K):
    """Segmented and plain prefill differ only in rounding (bf16 operand copies of
    M_p and of the incoming states)."""
    inp = case(1, 1024, 3, 128, 128, "bf16", seed=25, s0_std=0.1)
    o1, S1 = run_seg(K, inp, 64, 192)
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64)
    torch.cuda.synchronize()
    assert rel(to_f64(o1), to_f64(o2)) < 1e-2 and rel(to_f64(S1), to_f64(S2)) < 1e-2


def test_long_sequence_few_heads_sampled(K, oracle_mod):
    """The long-sequence workload (8 heads x 65536 tokens, 18 segments of 3648) in
    the launch configuration the benchmark times; two heads checked in full."""
    w = WORKLOADS["long_h8_T65536_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    o, ST = run_seg(K, inp, w.chunk, w.seg_len)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    units = [(0, 0), (0, 5)]
    o_ref, ST_ref = oracle_forward(oracle_mod, inp, units=units)
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, units, tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_pairs_scan_replay_by_hand(K, oracle_mod, path):
    """The context-parallel pieces on one GPU: three segments' pairs, the scan, and
    each segment replayed from its incoming state, against the oracle's single pass."""
    inp = case(2, 3 * 192 - 40, 2, 128, 128, "bf16", seed=71, s0_std=0.1)
    T = inp["k"].shape[1]
    cuts = [(0, 192), (192, 384), (384, T)]
    pairs = [K.kda_segment_pair(*(inp[x][:, a:b].contiguous() for x in ("q", "k", "v", "g", "beta")), path=path)
             for a, b in cuts]
    M = torch.stack([p[0] for p in pairs], 1)
    Z = torch.stack([p[1] for p in pairs], 1)
    S_in, S_T = K.kda_kcp_scan(inp["S0"], M, Z)
    o = torch.cat([K.kda_forward(*(inp[x][:, a:b].contiguous() for x in ("q", "k", "v", "g", "beta")),
                                 S_in[:, p].contiguous(), chunk=64, return_state=False, path=path)[0]
                   for p, (a, b) in enumerate(cuts)], 1)
    torch.cuda.synchronize()
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    e_o, e_s = compare_units(o, S_T, o_ref, ST_ref, [(b, h) for b in range(2) for h in range(2)], tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)


def test_context_parallel_module_one_rank_nccl(K):
    """The context-parallel module through a real NCCL group of one rank (the
    collective is the identity there): equals the plain prefill."""
    import torch.distributed as dist
    from linear_attention_recurrence_11_b200.context_parallel import context_parallel_forward
    inp = case(1, 320, 2, 128, 128, "bf16", seed=73, s0_std=0.1)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        o, S_T = context_parallel_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64)
    torch.cuda.synchronize()
    assert rel(to_f64(o), to_f64(o2)) < 1e-5 and rel(to_f64(S_T), to_f64(S2)) < 1e-2
