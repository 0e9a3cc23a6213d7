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


def run_seg_packed(K, inp, chunk, seg_len, path="auto"):
    status = torch.zeros(4, dtype=torch.int32, device=inp["k"].device)
    o, ST = K.kda_forward_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"),
                                    seg_len=seg_len, chunk=chunk, cu_seqlens=inp["cu_seqlens"], path=path,
                                    dev_status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0, f"device status {int(status[0])}"
    return o, ST


def packed_case(lens, H, dk, dv, dtype, seed, s0_std=0.1):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    inp = case(1, int(cu[-1]), H, dk, dv, dtype, seed=seed, s0_std=s0_std, num_states=len(lens))
    inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
    return inp, [int(x) for x in cu]


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("lens,seg_len", [([1, 65, 700, 0, 64, 300, 256], 128), ([900, 0, 3], 256),
                                          ([640], 64), ([500, 501], 192), ([0, 0, 130], 64)])
def test_packed_segments(K, oracle_mod, path, lens, seg_len):
    """Packed sequences, each cut into ceil(len / seg_len) segments (one for the short and
    the empty ones): ragged last segments and chunks, a length that is a multiple of
    seg_len, empty sequences (their state passes through bit for bit)."""
    H = 2
    inp, cu = packed_case(lens, H, 128, 128, "bf16", seed=sum(lens) + seg_len)
    o, ST = run_seg_packed(K, inp, 64, seg_len, path)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    units = [(n, h) for n in range(len(lens)) for h in range(H)]
    compare_units(o, ST, o_ref, ST_ref, units, cu, tol=TOL["bf16"], label=f"packed segments {path}")
    zero = [n for n, L in enumerate(lens) if L == 0]
    if zero:
        assert torch.equal(ST[zero], inp["S0"][zero])


@pytest.mark.parametrize("dtype,dk,dv,chunk,lens,seg_len", [
    ("f32", 32, 32, 16, [300, 17, 0, 96], 64), ("f32", 64, 128, 32, [257, 400], 96),
    ("bf16", 64, 32, 16, [33, 200, 64], 48)])
def test_packed_segments_simt_shapes(K, oracle_mod, dtype, dk, dv, chunk, lens, seg_len):
    inp, cu = packed_case(lens, 2, dk, dv, dtype, seed=dk + dv + seg_len)
    o, ST = run_seg_packed(K, inp, chunk, seg_len)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    units = [(n, h) for n in range(len(lens)) for h in range(2)]
    compare_units(o, ST, o_ref, ST_ref, units, cu, tol=TOL[dtype], label="packed segments simt shapes")


def test_packed_segments_uncut_is_the_plain_prefill(K):
    """T <= seg_len: no sequence is cut, the call is kda_forward_ex with cu_seqlens."""
    inp, cu = packed_case([100, 0, 200], 2, 128, 128, "bf16", seed=29)
    o1, S1 = run_seg_packed(K, inp, 64, 320)
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64,
                           cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_varlen_workload_segmented_sampled(K, oracle_mod):
    """The packed 8-sequence workload (96 heads, 352,549 tokens) through the
    segment-parallel prefill with 16,384-token segments (its two longest sequences
    become 6 and 7 segments; more (segment, head) units than three per SM, so the
    passes run the single-kernel prefill): oracle parity on units of the two longest
    sequences and of a short one, streamed over the host cores."""
    from kda_testutil import parity_streamed
    w = WORKLOADS["varlen_h96_8seq_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    o, ST = run_seg_packed(K, inp, w.chunk, 16384)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    lens = np.diff(inp["cu_seqlens"].cpu().numpy())
    order = [int(i) for i in np.argsort(-lens)]
    units = [(order[0], 0), (order[0], 95), (order[1], 47), (order[-1], 3)]
    parity_streamed(oracle_mod, inp, o, ST, units, TOL["bf16"], label="varlen segmented")
