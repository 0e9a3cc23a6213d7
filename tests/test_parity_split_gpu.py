"""GPU parity of the tensor-core prefill forms against each other and the
oracle: the split form (a chunk-parallel kernel writes every chunk's
state-independent operands to the workspace, a second kernel carries each
unit's state), the pipe form (both roles in one cooperative launch, records
through a ring) and the single-kernel form compute the same chunked recurrence
("Exercices", Q7, Q21-Q22) and must agree with the fp64 oracle and with each
other; the workspace passed decides which form AUTO runs."""
import numpy as np
import pytest
import torch

from kda_testutil import TOL, case, compare_units, oracle_forward, rel
from linear_attention_recurrence_11_b200.inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def fwd(K, inp, path, **kw):
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), chunk=64,
                          cu_seqlens=inp.get("cu_seqlens"), path=path, dev_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    return o, ST


FORMS = ["tc_split", "tc_pipe"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 200, 3), (1, 1, 2), (3, 127, 2), (1, 64 * 9 + 5, 4)])
def test_split_matches_oracle_and_single(K, oracle_mod, B, T, H, form):
    inp = case(B, T, H, 128, 128, "bf16", seed=1000 + T + B, s0_std=0.05, g_min_frac=0.1)
    o_s, S_s = fwd(K, inp, form)
    o_f, S_f = fwd(K, inp, "tc_single")
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    units = [(b, h) for b in range(B) for h in range(H)]
    compare_units(o_s, S_s, o_ref, S_ref, units, tol=TOL["bf16"], label="split")
    compare_units(o_f, S_f, o_ref, S_ref, units, tol=TOL["bf16"], label="single")
    # the two forms round at slightly different points (Ut reaches the state product in bf16
    # in the split form), so they agree to the bf16 level, not bit for bit
    assert rel(to_f64(o_s), to_f64(o_f)) < 5e-3 and rel(to_f64(S_s), to_f64(S_f)) < 5e-3


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("lens", [[1, 65, 130, 0, 64, 7, 200], [0, 0, 3], [500], [64] * 40 + [0, 129]])
def test_split_packed(K, oracle_mod, lens, form):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H = 3
    inp = case(1, int(cu[-1]), H, 128, 128, "bf16", seed=len(lens) + int(cu[-1]), s0_std=0.1,
               num_states=len(lens))
    inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
    o, ST = fwd(K, inp, form)
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    units = [(n, h) for n in range(len(lens)) for h in range(H)]
    compare_units(o, ST, o_ref, S_ref, units, cu, tol=TOL["bf16"], label=form + " packed")
    zero = [n for n, L in enumerate(lens) if L == 0]
    if zero:
        assert torch.equal(ST[zero], inp["S0"][zero])


@pytest.mark.parametrize("form", FORMS)
def test_split_identity_transition_is_exact(K, form):
    """beta = 0, g = 0: every record's W, Ut and P-columns vanish and Gamma_C = 1, so the
    state passes through bit for bit."""
    inp = case(2, 150, 2, 128, 128, "bf16", seed=21, s0_std=0.5)
    inp["g"].zero_(); inp["beta"].zero_()
    o, ST = fwd(K, inp, form)
    assert torch.equal(ST, inp["S0"])
    ref = torch.einsum("bthi,bhji->bthj", inp["q"].double(), inp["S0"].double())
    assert rel(to_f64(o), ref.cpu().numpy()) < TOL["bf16"]


@pytest.mark.parametrize("form", FORMS)
def test_split_g_min_runs(K, oracle_mod, form):
    """Whole channels and 128-token runs at g = g_min = -5 (the e^80 subtile bound)."""
    inp = case(1, 256, 2, 128, 128, "bf16", seed=11, s0_std=0.1)
    inp["g"][:, :, :, ::3] = -5.0
    inp["g"][:, 64:192] = -5.0
    o, ST = fwd(K, inp, form)
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    compare_units(o, ST, o_ref, S_ref, [(0, 0), (0, 1)], tol=TOL["bf16"], label="split g_min")


@pytest.mark.parametrize("spare", [8, 60])
def test_split_one_sequence_records_beside_the_chains(K, oracle_mod, spare):
    """One sequence whose heads leave `spare` SMs beside their chains: the prep kernel writes
    the first chunks' records and the last ones are produced on the spare SMs while the chains
    run (each chain waits for such a record by its flag). Sampled heads against the oracle,
    every head bit for bit against the pipe form (the same records and chain arithmetic), and
    a ragged last chunk."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = sms - spare
    inp = case(1, 64 * 11 + 37, H, 128, 128, "bf16", seed=90 + spare, s0_std=0.1, g_min_frac=0.1)
    o, ST = fwd(K, inp, "tc_split")
    units = [(0, h) for h in (0, 1, H // 2, H - 2, H - 1)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp, units=units)
    compare_units(o, ST, o_ref, S_ref, units, tol=TOL["bf16"], label=f"split, {spare} spare SMs")
    o_p, S_p = fwd(K, inp, "tc_pipe")
    assert torch.equal(o, o_p) and torch.equal(ST, S_p)


@pytest.mark.parametrize("T", [64 * 3 + 61, 64 * 2 + 61])
def test_split_one_sequence_fewest_heads(K, oracle_mod, T):
    """32 heads, the fewest that take the records-beside-chains launch. At 4 chunks (the fewest
    it takes) every chunk but the first is produced beside the chains, the ragged last one
    included; at 3 chunks the two-kernel form runs. Every head against the oracle, and bit for
    bit against the pipe form."""
    H = 32
    inp = case(1, T, H, 128, 128, "bf16", seed=95 + T, s0_std=0.1, g_min_frac=0.1)
    o, ST = fwd(K, inp, "tc_split")
    units = [(0, h) for h in range(H)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp, units=units)
    compare_units(o, ST, o_ref, S_ref, units, tol=TOL["bf16"], label=f"split, 32 heads, T={T}")
    o_p, S_p = fwd(K, inp, "tc_pipe")
    assert torch.equal(o, o_p) and torch.equal(ST, S_p)


def test_auto_dense_many_units_takes_split(K, oracle_mod):
    """A dense batch of more units than three per SM (5 x 96 = 480, under the eight per SM of
    dense batches): AUTO runs the split form, its chains in waves of one per SM. The same
    outputs as a forced split call bit for bit (the single kernel rounds differently), and
    sampled units against the oracle."""
    B, T, H = 5, 130, 96
    assert B * H > 3 * torch.cuda.get_device_properties(0).multi_processor_count
    inp = case(B, T, H, 128, 128, "bf16", seed=97, s0_std=0.05)
    o, ST = fwd(K, inp, "auto")
    o_s, S_s = fwd(K, inp, "tc_split")
    assert torch.equal(o, o_s) and torch.equal(ST, S_s)
    units = [(0, 0), (1, 17), (2, 50), (4, 95)]
    o_ref, S_ref = oracle_forward(oracle_mod, inp, units=units)
    compare_units(o, ST, o_ref, S_ref, units, tol=TOL["bf16"], label="auto, 480 dense units")


def test_split_one_sequence_in_a_cuda_graph(K):
    """The one-sequence split step (40 heads: a cooperative launch beside the prep kernel)
    captured in a CUDA graph and replayed: the same outputs as the eager call, bit for bit."""
    H = 40
    inp = case(1, 64 * 9 + 3, H, 128, 128, "bf16", seed=93, s0_std=0.1)
    o_e, S_e = fwd(K, inp, "tc_split")
    o = torch.empty_like(o_e)
    ST = torch.empty_like(S_e)
    ws = torch.empty(K.kda_forward_workspace_size(1, inp["k"].shape[1], H, 128, 128, 64, 1, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64, o=o, S_T=ST,
                      workspace=ws, path="tc_split")
    for _ in range(2):
        o.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_e) and torch.equal(ST, S_e)


def test_workspace_decides_the_form(K):
    """AUTO with the reported workspace runs the split form; with only the pipe form's ring it
    runs the pipe form; with a few bytes (or none) the single form; a forced form with too
    small a workspace is refused."""
    inp = case(1, 300, 2, 128, 128, "bf16", seed=5, s0_std=0.1)
    o_split, S_split = fwd(K, inp, "tc_split")
    o_pipe, S_pipe = fwd(K, inp, "tc_pipe")
    o_single, S_single = fwd(K, inp, "tc_single")
    o_a, S_a = fwd(K, inp, "auto")
    assert torch.equal(o_a, o_split) and torch.equal(S_a, S_split)
    # the two record forms compute the same records and the same chain: bit for bit
    assert torch.equal(o_pipe, o_split) and torch.equal(S_pipe, S_split)
    ring = torch.empty(2 * 4 * 74752 + 256, dtype=torch.uint8, device="cuda")
    o_r, S_r = fwd(K, inp, "auto", workspace=ring)
    assert torch.equal(o_r, o_pipe) and torch.equal(S_r, S_pipe)
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    o_b, S_b = fwd(K, inp, "auto", workspace=small)
    assert torch.equal(o_b, o_single) and torch.equal(S_b, S_single)
    for form in FORMS:
        with pytest.raises(K.KdaError) as e:
            fwd(K, inp, form, workspace=small)
        assert e.value.code == K.KDA_ERR_WORKSPACE


@pytest.mark.parametrize("form", ["auto", "tc_pipe"])
def test_split_two_calls_reuse_workspace(K, oracle_mod, form):
    """The records are scratch: a second call with other inputs in the same workspace gives
    its own results (every record is rewritten before it is read, the ring's flags are
    reset by every call)."""
    ws = torch.empty(K.kda_forward_workspace_size(2, 256, 2, 128, 128, 64, 2, torch.bfloat16, path=form),
                     dtype=torch.uint8, device="cuda")
    for seed in (1, 2):
        inp = case(2, 256, 2, 128, 128, "bf16", seed=seed, s0_std=0.1)
        o, ST = fwd(K, inp, form, workspace=ws)
        o_ref, S_ref = oracle_forward(oracle_mod, inp)
        compare_units(o, ST, o_ref, S_ref, [(b, h) for b in range(2) for h in range(2)], tol=TOL["bf16"])


@pytest.mark.parametrize("B,T,H,lens", [(3, 130, 70, None), (1, 0, 6, [64] * 40 + [0, 129])])
def test_split_two_kernel_form(K, oracle_mod, B, T, H, lens):
    """More (sequence, head) units than the one-launch form takes (two thirds of two CTAs per
    SM): every chunk's record goes to the workspace, then the chains run (dense and packed)."""
    if lens is None:
        inp = case(B, T, H, 128, 128, "bf16", seed=77, s0_std=0.05)
        units = [(b, h) for b in range(B) for h in range(H)]
        cu = None
    else:
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        inp = case(1, int(cu[-1]), H, 128, 128, "bf16", seed=78, s0_std=0.05, num_states=len(lens))
        inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
        units = [(n, h) for n in range(len(lens)) for h in range(H)]
    assert len(units) * 3 > 2 * 2 * torch.cuda.get_device_properties(0).multi_processor_count
    o, ST = fwd(K, inp, "tc_split")
    o_ref, S_ref = oracle_forward(oracle_mod, inp, units=units)
    compare_units(o, ST, o_ref, S_ref, units, cu, tol=TOL["bf16"], label="split two-kernel")
