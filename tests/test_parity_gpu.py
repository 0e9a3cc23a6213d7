"""GPU parity: libkda.so (through the C ABI) against the fp64 oracle on the same
seeded inputs. Tolerances (normwise relative error per output tensor): 1e-4
for fp32 inputs, 1e-2 for bf16 inputs against the oracle fed the identical
bf16-rounded values."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_11_b200.inputs import WORKLOADS, make_inputs, to_f64, workload_inputs

from kda_testutil import TOL, case, compare_units, oracle_forward, parity_streamed, rel

pytestmark = pytest.mark.gpu

# "auto" runs the split tensor-core form on its shapes (the wrapper passes the workspace it
# reports) and SIMT elsewhere; "tc_single" forces the single-kernel tensor-core form.
PATHS = ["simt", "auto", "tc_single"]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def run(K, inp, chunk, path="auto", **kw):
    if path.startswith("tc_"):
        B, T, H, dk = inp["k"].shape
        if K.kda_forward_launches(B, T, H, dk, inp["v"].shape[-1], chunk, inp["k"].dtype,
                                  inp.get("cu_seqlens") is not None, 1, path) < 0:
            pytest.skip("shape outside the tensor-core kernels")
    status = torch.zeros(4, dtype=torch.int32, device=inp["k"].device)
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"),
                          chunk=chunk, cu_seqlens=inp.get("cu_seqlens"), path=path,
                          dev_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status[0]) == 0, f"device status {int(status[0])}"
    return o, ST


def all_units(N, H):
    return [(n, h) for n in range(N) for h in range(H)]


def check_full(K, oracle_mod, inp, chunk, dtype, path, cu=None):
    o, ST = run(K, inp, chunk, path)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    N, H = ST.shape[0], ST.shape[1]
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, all_units(N, H), cu, tol=TOL[dtype])
    assert e_o < TOL[dtype] and e_s < TOL[dtype], (e_o, e_s)
    return e_o, e_s


@pytest.mark.parametrize("path", PATHS)
def test_small_fp32_workload(K, oracle_mod, path):
    w = WORKLOADS["small_f32_T256_d32"]
    inp = workload_inputs(w, device="cuda")
    check_full(K, oracle_mod, inp, w.chunk, "f32", path)


@pytest.mark.parametrize("path", PATHS)
def test_b2_h4_T2048_bf16_workload(K, oracle_mod, path):
    w = WORKLOADS["b2_h4_T2048_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    check_full(K, oracle_mod, inp, w.chunk, "bf16", path)


@pytest.mark.parametrize("dtype,dk,dv,chunk,T", [
    ("f32", 128, 128, 64, 200), ("f32", 64, 32, 32, 77), ("f32", 32, 64, 16, 5),
    ("bf16", 128, 128, 64, 200), ("bf16", 128, 128, 64, 64 * 5 + 1), ("bf16", 64, 128, 16, 33),
    ("bf16", 128, 128, 64, 1), ("bf16", 128, 128, 64, 15),
])
@pytest.mark.parametrize("path", PATHS)
def test_ragged_shapes(K, oracle_mod, dtype, dk, dv, chunk, T, path):
    inp = case(2, T, 3, dk, dv, dtype, seed=T * 7 + dk + dv, s0_std=0.1)
    check_full(K, oracle_mod, inp, chunk, dtype, path)


@pytest.mark.parametrize("path", PATHS)
def test_varlen_with_edge_lengths(K, oracle_mod, path):
    lens = [1, 65, 130, 0, 64, 7, 200]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    inp = case(1, int(cu[-1]), 2, 128, 128, "bf16", seed=5, s0_std=0.1, num_states=len(lens))
    inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
    o, ST = run(K, inp, 64, path)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, all_units(len(lens), 2), cu, tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)
    # the empty sequence passes its state through untouched
    assert torch.equal(ST[3], inp["S0"][3])


@pytest.mark.parametrize("nseq", [40, 2100])
def test_varlen_many_sequences(K, oracle_mod, nseq):
    """Many packed sequences of mixed lengths (zeros included): with up to 2048
    sequences a longest-first schedule runs first; above that, natural order."""
    rng = np.random.default_rng(nseq)
    if nseq <= 2048:
        lens = rng.integers(0, 300, size=nseq)
    else:
        lens = rng.integers(0, 4, size=nseq)
    lens[::7] = 0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H = 2
    inp = case(1, int(cu[-1]), H, 128, 128, "bf16", seed=nseq, s0_std=0.1, num_states=nseq)
    inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
    o, ST = run(K, inp, 64, "auto")
    picks = [int(i) for i in np.argsort(-lens)[:3]] + [int(np.argmin(lens)), nseq - 1]
    units = [(n, h) for n in picks for h in range(H)]
    o_ref, ST_ref = oracle_forward(oracle_mod, inp, units=units)
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, units, cu, tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)
    zero = np.nonzero(lens == 0)[0]
    assert torch.equal(ST[zero], inp["S0"][zero])


@pytest.mark.parametrize("path", PATHS)
def test_identity_transition_is_exact(K, path):
    """beta = 0, g = 0: S_T = S0 bit for bit and o_t = S0^T q_t."""
    inp = case(1, 130, 2, 128, 128, "bf16", seed=9, s0_std=0.5)
    inp["g"].zero_(); inp["beta"].zero_()
    o, ST = run(K, inp, 64, path)
    assert torch.equal(ST, inp["S0"])
    ref = torch.einsum("bthi,bhji->bthj", inp["q"].double(), inp["S0"].double())
    assert rel(to_f64(o), ref.cpu().numpy()) < TOL["bf16"]


@pytest.mark.parametrize("path", PATHS)
def test_g_min_runs(K, oracle_mod, path):
    """Whole channels at g = g_min = -5 for >= 64 tokens (the e^80 subtile bound)."""
    inp = case(1, 256, 2, 128, 128, "bf16", seed=11, s0_std=0.1)
    inp["g"][:, :, :, ::3] = -5.0
    inp["g"][:, 64:192] = -5.0
    check_full(K, oracle_mod, inp, 64, "bf16", path)


@pytest.mark.parametrize("path", PATHS)
def test_s0_none_equals_zeros_and_state_in_place(K, path):
    inp = case(2, 100, 2, 128, 128, "bf16", seed=13)
    o1, S1 = run(K, inp, 64, path)
    inp2 = dict(inp); inp2["S0"] = torch.zeros_like(S1)
    o2, S2 = run(K, inp2, 64, path)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    # S_T may alias S0
    S = torch.randn_like(S1) * 0.1
    o3, S3 = run(K, dict(inp, S0=S.clone()), 64, path)
    Sa = S.clone()
    o4, _ = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], Sa, chunk=64,
                          S_T=Sa, path=path)
    torch.cuda.synchronize()
    assert torch.equal(o3, o4) and torch.equal(S3, Sa)


@pytest.mark.parametrize("path", PATHS)
def test_chaining_two_calls_equals_one(K, path):
    """The S0 -> S_T interface is a checkpoint: two calls = one call."""
    inp = case(1, 256, 2, 128, 128, "bf16", seed=17, s0_std=0.1)
    o, ST = run(K, inp, 64, path)
    a = {k: (v[:, :128].contiguous() if k in "qkvg" or k == "beta" else v) for k, v in inp.items()}
    b = {k: (v[:, 128:].contiguous() if k in "qkvg" or k == "beta" else v) for k, v in inp.items()}
    oa, Sm = run(K, a, 64, path)
    b["S0"] = Sm
    ob, S2 = run(K, b, 64, path)
    # chunk boundaries line up (128 = 2 chunks), so the two paths agree closely
    assert rel(to_f64(torch.cat([oa, ob], 1)), to_f64(o)) < 1e-5
    assert rel(to_f64(S2), to_f64(ST)) < 1e-5


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("dtype,dk,dv", [("f32", 128, 128), ("bf16", 128, 128), ("f32", 32, 64),
                                         ("bf16", 64, 32)])
def test_decode_steps(K, oracle_mod, dtype, dk, dv):
    N, H, steps = 5, 3, 6
    S = (0.02 * torch.randn(N, H, dv, dk, generator=torch.Generator().manual_seed(1))).cuda()
    S_ref = to_f64(S)
    for t in range(steps):
        inp = make_inputs(N, 1, H, dk, dv, dtype, seed=100 + t, device="cuda")
        d = {k: inp[k][:, 0].contiguous() for k in ("q", "k", "v", "g", "beta")}
        o = K.kda_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S)
        torch.cuda.synchronize()
        hd = {k: to_f64(v) for k, v in d.items()}
        o_ref = np.empty((N, H, dv))
        for n in range(N):
            for h in range(H):
                St = np.ascontiguousarray(S_ref[n, h])
                o_ref[n, h] = oracle_mod.decode_step(hd["q"][n, h], hd["k"][n, h], hd["v"][n, h],
                                                     hd["g"][n, h], hd["beta"][n, h], St)
                S_ref[n, h] = St
        assert rel(to_f64(o), o_ref) < TOL[dtype]
        assert rel(to_f64(S), S_ref) < TOL[dtype]


def test_decode_full_size_1000_steps_sampled(K, oracle_mod):
    """256 requests x 96 heads, 1000 steps on the GPU, states in place. Eight
    seeded (request, head) pairs are followed by the oracle through all 1000
    steps; after step 1 every one of the 24,576 (request, head) pairs is checked
    (state and output, pooled and worst pair)."""
    w = WORKLOADS["decode_n256_h96_d128"]
    rng = np.random.default_rng(0)
    picks = [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(8)]
    pn, ph = [p[0] for p in picks], [p[1] for p in picks]
    inp0 = workload_inputs(w, device="cuda", step=0)
    S = inp0["S0"]
    S_init = to_f64(S)
    refs = [S_init[n, h].copy() for n, h in picks]  # copies: the oracle steps them in place
    for t in range(w.decode_steps):
        inp = inp0 if t == 0 else workload_inputs(w, device="cuda", step=t)
        d = {k: inp[k][:, 0].contiguous() for k in ("q", "k", "v", "g", "beta")}
        o = K.kda_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S)
        sub = {k: to_f64(d[k][pn, ph]) for k in d}
        o_ref = np.stack([oracle_mod.decode_step(sub["q"][i], sub["k"][i], sub["v"][i],
                                                 sub["g"][i], sub["beta"][i], refs[i])
                          for i in range(len(picks))])
        if t == 0:
            hd = {k: to_f64(v) for k, v in d.items()}
            S1 = to_f64(S)
            o1 = to_f64(o)
            num = den = onum = oden = 0.0
            worst_s = worst_o = 0.0
            for n in range(w.B):
                for h in range(w.H):
                    St = S_init[n, h].copy()
                    ot = oracle_mod.decode_step(hd["q"][n, h], hd["k"][n, h], hd["v"][n, h],
                                                hd["g"][n, h], hd["beta"][n, h], St)
                    es, ds = np.sum((S1[n, h] - St) ** 2), np.sum(St ** 2)
                    eo, do = np.sum((o1[n, h] - ot) ** 2), np.sum(ot ** 2)
                    num += es; den += ds; onum += eo; oden += do
                    worst_s = max(worst_s, np.sqrt(es / ds))
                    worst_o = max(worst_o, np.sqrt(eo / do) if do > 0 else 0.0)
            print(f"[parity decode step 1] pairs={w.B * w.H} S={np.sqrt(num / den):.3e} o={np.sqrt(onum / oden):.3e} "
                  f"worst S={worst_s:.3e} worst o={worst_o:.3e}")
            assert np.sqrt(num / den) < TOL["bf16"] and worst_s < TOL["bf16"]
            assert np.sqrt(onum / oden) < TOL["bf16"] and worst_o < TOL["bf16"]
            del S1, o1
        if t == w.decode_steps - 1:
            assert rel(to_f64(o[pn, ph]), o_ref) < TOL["bf16"]
    Sg = to_f64(S)
    assert rel(np.stack([Sg[n, h] for n, h in picks]), np.stack(refs)) < TOL["bf16"]


# ------------------------------------------------------- full-size prefill

def test_prefill_h96_T8192_all_heads(K, oracle_mod):
    """The layer-shape workload at full size, in the launch configuration the
    benchmark times: every one of the 96 heads recomputed by the oracle in
    full (on all host cores), the pooled and the worst per-head error gated."""
    w = WORKLOADS["prefill_h96_T8192_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    o, ST = run(K, inp, w.chunk, "auto")
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    parity_streamed(oracle_mod, inp, o, ST, all_units(1, w.H), TOL["bf16"], label="h96_T8192")


def test_varlen_full_size_sampled(K, oracle_mod):
    """Eight packed long sequences (log-uniform lengths in [4096, 131072]); the
    oracle follows at least one head of every sequence end to end (a different
    head for each), plus two more heads of the longest and the shortest."""
    w = WORKLOADS["varlen_h96_8seq_d128_bf16"]
    inp = workload_inputs(w, device="cuda")
    o, ST = run(K, inp, w.chunk, "auto")
    assert torch.isfinite(ST).all()
    order = sorted(range(w.num_seqs), key=lambda n: w.seqlens[n])
    units = [(n, (13 * n + 5) % w.H) for n in range(w.num_seqs)]
    units += [(order[0], 60), (order[-1], 17)]
    parity_streamed(oracle_mod, inp, o, ST, units, TOL["bf16"], label="varlen_8seq")
