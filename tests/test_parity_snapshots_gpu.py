"""GPU parity of the prefill state snapshots (every snap_every tokens, the state
after that prefix) against the fp64 oracle run on the prefixes, through the C ABI."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_11_b200.inputs import to_f64

from kda_testutil import TOL, case, compare_units, oracle_forward, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def prefix_states(oracle_mod, inp, b, h, ends):
    a = [to_f64(inp[x][b, :, h]) for x in ("q", "k", "v", "g", "beta")]
    s0 = None if inp.get("S0") is None else to_f64(inp["S0"][b, h])
    return [oracle_mod.forward(*[x[:e] for x in a], S0=s0)[1] for e in ends]


@pytest.mark.parametrize("dtype,dk,dv,chunk,T,every,path", [
    ("bf16", 128, 128, 64, 1000, 256, "auto"), ("bf16", 128, 128, 64, 1000, 256, "simt"),
    ("bf16", 128, 128, 64, 1000, 256, "tc_single"), ("bf16", 128, 128, 64, 512, 64, "tc_split"),
    ("bf16", 128, 128, 64, 512, 64, "auto"), ("f32", 32, 32, 16, 256, 48, "auto"),
    ("f32", 64, 128, 32, 300, 96, "auto"),
])
def test_snapshots(K, oracle_mod, dtype, dk, dv, chunk, T, every, path):
    B, H = 2, 2
    inp = case(B, T, H, dk, dv, dtype, seed=T + every + dk, s0_std=0.1)
    o, ST, Ssn = K.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"],
                                         snap_every=every, chunk=chunk, path=path)
    torch.cuda.synchronize()
    ns = T // every
    assert Ssn.shape == (B, ns, H, dv, dk)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, [(b, h) for b in range(B) for h in range(H)], tol=TOL[dtype])
    assert e_o < TOL[dtype] and e_s < TOL[dtype], (e_o, e_s)
    for b in range(B):
        for h in range(H):
            refs = prefix_states(oracle_mod, inp, b, h, [(p + 1) * every for p in range(ns)])
            got = to_f64(Ssn[b, :, h])
            assert rel(got, np.stack(refs)) < TOL[dtype]


def test_snapshots_one_sequence_split_form(K, oracle_mod):
    """One sequence of 40 heads on the split form: the chains store their snapshots while the
    last chunks' records are produced beside them (sampled heads against the oracle)."""
    T, H, every = 64 * 14 + 21, 40, 128
    inp = case(1, T, H, 128, 128, "bf16", seed=67, s0_std=0.1)
    o, ST, Ssn = K.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"],
                                         snap_every=every, chunk=64, path="tc_split")
    torch.cuda.synchronize()
    ns = T // every
    heads = (0, 1, H // 2, H - 1)
    o_ref, ST_ref = oracle_forward(oracle_mod, inp, units=[(0, h) for h in heads])
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, [(0, h) for h in heads], tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"], (e_o, e_s)
    for h in heads:
        refs = prefix_states(oracle_mod, inp, 0, h, [(p + 1) * every for p in range(ns)])
        assert rel(to_f64(Ssn[0, :, h]), np.stack(refs)) < TOL["bf16"], h


@pytest.mark.parametrize("path", ["auto", "tc_single"])
def test_resume_from_a_snapshot(K, path):
    """A snapshot is a valid S0: resuming from it on the same form reproduces the rest of
    the run (the split form's chains and the single kernel both save the fp32 state they
    carry)."""
    inp = case(1, 768, 2, 128, 128, "bf16", seed=61, s0_std=0.1)
    o, ST, Ssn = K.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"],
                                         snap_every=256, chunk=64, path=path)
    rest = {x: inp[x][:, 512:].contiguous() for x in ("q", "k", "v", "g", "beta")}
    o2, S2 = K.kda_forward(rest["q"], rest["k"], rest["v"], rest["g"], rest["beta"], Ssn[:, 1].contiguous(),
                           chunk=64, path=path)
    torch.cuda.synchronize()
    assert rel(to_f64(o2), to_f64(o[:, 512:])) < 1e-5 and rel(to_f64(S2), to_f64(ST)) < 1e-5


@pytest.mark.parametrize("path", ["auto", "tc_single"])
def test_no_snapshot_due(K, oracle_mod, path):
    """T < snap_every: no snapshot, the plain prefill results of the same form."""
    inp = case(1, 100, 2, 128, 128, "bf16", seed=63)
    o, ST, Ssn = K.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None,
                                         snap_every=128, chunk=64, path=path)
    o2, S2 = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, chunk=64, path=path)
    torch.cuda.synchronize()
    assert Ssn.shape[1] == 0 and torch.equal(o, o2) and torch.equal(ST, S2)


def test_snapshots_refused_on_the_pipe_form(K):
    inp = case(1, 256, 2, 128, 128, "bf16", seed=65)
    with pytest.raises(K.KdaError):
        K.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, snap_every=128,
                                chunk=64, path="tc_pipe")
