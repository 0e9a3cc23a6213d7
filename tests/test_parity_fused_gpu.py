"""GPU parity of the fused pre-operations (raw q and k normalised per row inside
the kernels; g given as gate logits x, log-decay g_min sigmoid(x)) against the
fp64 oracle fed the normalised rows and the decays computed in fp64 from the
same rounded raw inputs."""
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


def raw_inputs(B, T, H, dk, dv, dtype, seed):
    """Unnormalised q, k (rows scaled by factors in [0.3, 3], a few all-zero rows)
    and gate logits ~ N(0, 1.5^2)."""
    inp = make_inputs(B, T, H, dk, dv, dtype, seed=seed, device="cuda", s0_std=0.1)
    gen = torch.Generator(device="cuda").manual_seed(seed + 1)
    for x in ("q", "k"):
        sc = 0.3 + 2.7 * torch.rand((B, T, H, 1), generator=gen, device="cuda")
        inp[x] = (inp[x].float() * sc).to(inp[x].dtype)
    inp["k"][:, ::37] = 0
    inp["g"] = (1.5 * torch.randn(inp["g"].shape, generator=gen, device="cuda")).to(inp["g"].dtype)
    return inp


def reference_inputs(inp):
    """fp64 arrays the oracle takes: normalised rows (zero rows stay zero) and decays."""
    out = {}
    for x in ("q", "k"):
        a = to_f64(inp[x])
        n = np.linalg.norm(a, axis=-1, keepdims=True)
        out[x] = np.divide(a, n, out=np.zeros_like(a), where=n > 0)
    out["g"] = -5.0 / (1.0 + np.exp(-to_f64(inp["g"])))
    out["v"], out["beta"] = to_f64(inp["v"]), to_f64(inp["beta"])
    return out


@pytest.mark.parametrize("dtype,dk,dv,chunk,T,path", [
    ("bf16", 128, 128, 64, 300, "auto"), ("bf16", 128, 128, 64, 300, "simt"), ("f32", 64, 32, 32, 150, "auto"),
    ("bf16", 32, 64, 16, 100, "auto"), ("bf16", 128, 128, 64, 300, "tc_split"),
    ("bf16", 128, 128, 64, 300, "tc_single"),
])
def test_fused_prefill(K, oracle_mod, dtype, dk, dv, chunk, T, path):
    B, H = 2, 2
    inp = raw_inputs(B, T, H, dk, dv, dtype, seed=T + dk)
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=chunk, path=path,
                          fuse=K.KDA_FUSE_NORM_QK | K.KDA_FUSE_GATE_LOGITS)
    torch.cuda.synchronize()
    r = reference_inputs(inp)
    S0 = to_f64(inp["S0"])
    o_ref = np.empty(o.shape); S_ref = np.empty(ST.shape)
    for b in range(B):
        for h in range(H):
            ou, su = oracle_mod.forward(*(r[x][b, :, h] for x in ("q", "k", "v", "g", "beta")), S0=S0[b, h])
            o_ref[b, :, h], S_ref[b, h] = ou, su
    assert rel(to_f64(o), o_ref) < TOL[dtype]
    assert rel(to_f64(ST), S_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_decode(K, oracle_mod, dtype):
    N, H, d = 4, 3, 128
    inp = raw_inputs(N, 1, H, d, d, dtype, seed=91)
    S = inp["S0"].clone()
    dd = {x: inp[x][:, 0].contiguous() for x in ("q", "k", "v", "g", "beta")}
    o = K.kda_decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S,
                          fuse=K.KDA_FUSE_NORM_QK | K.KDA_FUSE_GATE_LOGITS)
    torch.cuda.synchronize()
    r = reference_inputs(inp)
    S_ref = to_f64(inp["S0"])
    o_ref = np.empty((N, H, d))
    for n in range(N):
        for h in range(H):
            St = np.ascontiguousarray(S_ref[n, h])
            o_ref[n, h] = oracle_mod.decode_step(*(r[x][n, 0, h] for x in ("q", "k", "v", "g", "beta")), St)
            S_ref[n, h] = St
    assert rel(to_f64(o), o_ref) < TOL[dtype]
    assert rel(to_f64(S), S_ref) < TOL[dtype]


def test_fused_one_sequence_split_form(K, oracle_mod):
    """One sequence of 40 heads on the split form: the producers of the last chunks' records,
    beside the chains, apply the fused pre-operations too."""
    B, T, H = 1, 64 * 12 + 9, 40
    inp = raw_inputs(B, T, H, 128, 128, "bf16", seed=71)
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64,
                          path="tc_split", fuse=K.KDA_FUSE_NORM_QK | K.KDA_FUSE_GATE_LOGITS)
    torch.cuda.synchronize()
    r = reference_inputs(inp)
    S0 = to_f64(inp["S0"])
    for h in range(H):
        ou, su = oracle_mod.forward(*(r[x][0, :, h] for x in ("q", "k", "v", "g", "beta")), S0=S0[0, h])
        assert rel(to_f64(o[0, :, h]), ou) < TOL["bf16"] and rel(to_f64(ST[0, h]), su) < TOL["bf16"], h


def test_unfused_call_is_unchanged(K):
    """fuse = 0 takes the plain entry point (normalised inputs, g as log-decays)."""
    inp = make_inputs(1, 200, 2, 128, 128, "bf16", seed=93, device="cuda")
    o1, S1 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, chunk=64)
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, chunk=64, fuse=0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("flags", ["norm", "gate"])
def test_fused_packed_split_form(K, oracle_mod, flags):
    """Packed sequences through the split form's record producer with one fused
    pre-operation at a time (the other input given as the plain entry points take it)."""
    lens = [130, 0, 64, 257]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H = 2
    inp = raw_inputs(1, int(cu[-1]), H, 128, 128, "bf16", seed=97)
    S0 = (0.1 * torch.randn(len(lens), H, 128, 128, generator=torch.Generator().manual_seed(5))).cuda()
    r = reference_inputs(inp)
    if flags == "norm":
        f = K.KDA_FUSE_NORM_QK
        g_in = (-5.0 * torch.sigmoid(inp["g"].float())).to(inp["g"].dtype)
        r["g"] = to_f64(g_in)
    else:
        f = K.KDA_FUSE_GATE_LOGITS
        g_in = inp["g"]
        for x in ("q", "k"):
            inp[x] = torch.nn.functional.normalize(inp[x].float(), dim=-1).to(inp[x].dtype)
            r[x] = to_f64(inp[x])
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], g_in, inp["beta"], S0, chunk=64,
                          cu_seqlens=torch.tensor(cu, device="cuda"), path="tc_split", fuse=f)
    torch.cuda.synchronize()
    S0f = to_f64(S0)
    for n in range(len(lens)):
        for h in range(H):
            a, b = int(cu[n]), int(cu[n + 1])
            ou, su = oracle_mod.forward(*(r[x][0, a:b, h] for x in ("q", "k", "v", "g", "beta")), S0=S0f[n, h])
            if b > a:
                assert rel(to_f64(o[0, a:b, h]), ou) < TOL["bf16"], (n, h)
            assert rel(to_f64(ST[n, h]), su) < TOL["bf16"], (n, h)
