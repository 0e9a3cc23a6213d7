"""Failure detection on the GPU without a fault: a kernel waits (bounded) on an
mbarrier that nothing arrives on, through the same helper as every mbarrier
wait of the tensor-core prefill, and on a flag in global memory that nothing
sets, through the same helper as a chain waiting for a record produced beside
it; it must give up on both, report KDA_ERR_TIMEOUT for each and leave the
context usable for the next call."""
import pytest
import torch

from kda_testutil import TOL, case, compare_units, oracle_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def test_wait_runs_out_and_reports(K, oracle_mod):
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    K.kda_selftest_wait_timeout(status, max_cycles=20_000_000)  # ~10 ms of SM clocks per wait
    torch.cuda.synchronize()
    assert int(status[0]) == K.KDA_ERR_TIMEOUT  # the mbarrier wait
    assert int(status[1]) == 0 and int(status[2]) == K.KDA_ERR_TIMEOUT  # the flag wait
    # the context is intact: a prefill right after runs and matches the oracle
    inp = case(1, 200, 2, 128, 128, "bf16", seed=81, s0_std=0.1)
    st2 = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=64,
                          dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2[0]) == 0
    o_ref, ST_ref = oracle_forward(oracle_mod, inp)
    e_o, e_s = compare_units(o, ST, o_ref, ST_ref, [(0, 0), (0, 1)], tol=TOL["bf16"])
    assert e_o < TOL["bf16"] and e_s < TOL["bf16"]


def test_selftest_rejects_bad_arguments(K):
    with pytest.raises(K.KdaError):
        K.kda_selftest_wait_timeout(torch.zeros(4, dtype=torch.int32, device="cuda"), max_cycles=0)
