"""GPU parity of the multi-token decode with speculative acceptance against the
fp64 oracle's sequential decode steps, through the C ABI: outputs of all T
tokens, and the state after each request's accepted prefix."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_11_b200.inputs import make_inputs, to_f64

from kda_testutil import TOL, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def oracle_multi(oracle_mod, inp, S, n_acc):
    """Sequential oracle decode steps: outputs of all T tokens per request and the
    state after the first n_acc[n] tokens."""
    N, T, H, _ = inp["k"].shape
    dv = inp["v"].shape[-1]
    hd = {x: to_f64(inp[x]) for x in ("q", "k", "v", "g", "beta")}
    S0 = to_f64(S)
    o = np.empty((N, T, H, dv))
    S_out = S0.copy()
    for n in range(N):
        for h in range(H):
            St = np.ascontiguousarray(S0[n, h])
            for t in range(T):
                o[n, t, h] = oracle_mod.decode_step(hd["q"][n, t, h], hd["k"][n, t, h], hd["v"][n, t, h],
                                                    hd["g"][n, t, h], hd["beta"][n, t, h], St)
                if t + 1 == n_acc[n]:
                    S_out[n, h] = St
    return o, S_out


@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 128, 128, 4), ("f32", 128, 128, 8), ("bf16", 64, 32, 3),
                                           ("f32", 32, 64, 16), ("bf16", 128, 128, 64)])
def test_multi_token_with_acceptance(K, oracle_mod, dtype, dk, dv, T):
    N, H = 6, 3
    inp = make_inputs(N, T, H, dk, dv, dtype, seed=T * 13 + dk + dv, device="cuda")
    S = (0.02 * torch.randn(N, H, dv, dk, generator=torch.Generator().manual_seed(T))).cuda()
    n_acc = np.array([0, T, 1, T // 2, T - 1, 2 % (T + 1)], dtype=np.int32)
    o_ref, S_ref = oracle_multi(oracle_mod, inp, S, n_acc)
    acc = torch.tensor(n_acc, device="cuda")
    o = K.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S, n_accept=acc)
    torch.cuda.synchronize()
    assert rel(to_f64(o), o_ref) < TOL[dtype]
    assert rel(to_f64(S), S_ref) < TOL[dtype]
    # requests with nothing accepted keep their state bit for bit
    assert np.array_equal(to_f64(S[0]), S_ref[0])


def test_one_token_is_the_decode_step(K):
    N, H = 4, 5
    inp = make_inputs(N, 1, H, 128, 128, "bf16", seed=31, device="cuda")
    S1 = (0.02 * torch.randn(N, H, 128, 128, generator=torch.Generator().manual_seed(3))).cuda()
    S2 = S1.clone()
    o1 = K.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S1)
    d = {x: inp[x][:, 0].contiguous() for x in ("q", "k", "v", "g", "beta")}
    o2 = K.kda_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S2)
    torch.cuda.synchronize()
    assert rel(to_f64(o1[:, 0]), to_f64(o2)) < 1e-6 and rel(to_f64(S1), to_f64(S2)) < 1e-6


def test_verify_then_commit(K, oracle_mod):
    """Verification (outputs only, states untouched), then the commit of the accepted
    prefixes without outputs: the states equal those after the accepted tokens."""
    N, T, H = 8, 5, 2
    inp = make_inputs(N, T, H, 128, 128, "bf16", seed=41, device="cuda")
    S = (0.02 * torch.randn(N, H, 128, 128, generator=torch.Generator().manual_seed(5))).cuda()
    S_before = S.clone()
    zeros = torch.zeros(N, dtype=torch.int32, device="cuda")
    o = K.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S, n_accept=zeros)
    torch.cuda.synchronize()
    assert torch.equal(S, S_before)
    n_acc = np.random.default_rng(0).integers(0, T + 1, size=N).astype(np.int32)
    o_ref, S_ref = oracle_multi(oracle_mod, inp, S_before, n_acc)
    assert rel(to_f64(o), o_ref) < TOL["bf16"]
    assert K.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S,
                              n_accept=torch.tensor(n_acc, device="cuda"), outputs=False) is None
    torch.cuda.synchronize()
    assert rel(to_f64(S), S_ref) < TOL["bf16"]


def test_commit_without_outputs_equals_the_full_call(K):
    """Without outputs only the accepted tokens are applied (and a request with
    none accepted reads nothing): the states equal, bit for bit, those of the
    call that also produces every output; the status word stays clear."""
    N, T, H = 7, 6, 3
    inp = make_inputs(N, T, H, 128, 64, "bf16", seed=43, device="cuda")
    S1 = (0.02 * torch.randn(N, H, 64, 128, generator=torch.Generator().manual_seed(7))).cuda()
    S2 = S1.clone()
    acc = torch.tensor([0, 1, 2, 3, 6, 5, 4], dtype=torch.int32, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    args = [inp[x] for x in ("q", "k", "v", "g", "beta")]
    K.kda_decode_multi(*args, S1, n_accept=acc, dev_status=status)
    assert K.kda_decode_multi(*args, S2, n_accept=acc, outputs=False, dev_status=status) is None
    torch.cuda.synchronize()
    assert torch.equal(S1, S2) and int(status[0]) == 0


@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 128, 128, 1), ("bf16", 128, 128, 2), ("f32", 128, 128, 5),
                                           ("bf16", 64, 128, 7), ("f32", 32, 32, 13), ("bf16", 128, 64, 16),
                                           ("f32", 64, 64, 16), ("bf16", 128, 128, 17)])
def test_verification_form(K, oracle_mod, dtype, dk, dv, T):
    """Verification calls (outputs of all T tokens, nothing accepted): up to 16 tokens they
    take the chunked form (dot products of every state column with the decayed k_t and
    q_t, then T x T systems per column), beyond it the sequential steps; both against the
    oracle's sequential steps, with g at g_min on whole channels, and the states untouched."""
    N, H = 5, 3
    inp = make_inputs(N, T, H, dk, dv, dtype, seed=7 * T + dk + dv, device="cuda")
    g = inp["g"].clone()
    g[..., : dk // 4] = -5.0
    inp["g"] = g
    S = (0.05 * torch.randn(N, H, dv, dk, generator=torch.Generator().manual_seed(T + 100))).cuda()
    S_before = S.clone()
    zeros = np.zeros(N, dtype=np.int32)
    o_ref, _ = oracle_multi(oracle_mod, inp, S, zeros)
    o = K.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S,
                           n_accept=torch.tensor(zeros, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(S, S_before)
    worst = max(rel(to_f64(o[n, :, h]), o_ref[n, :, h]) for n in range(N) for h in range(H))
    assert worst < TOL[dtype], worst
