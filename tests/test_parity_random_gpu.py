"""Seeded random prefill cases against the fp64 oracle: the form (AUTO, each
tensor-core form, SIMT), dense or packed batches, sequence lengths around the
chunk size (1, 63, 64, 65, ...), with and without S0, decays pinned at g_min on
whole channels; every (sequence, head) unit gated on its own error."""
import numpy as np
import pytest
import torch

from kda_testutil import TOL, case, compare_units, oracle_forward

pytestmark = pytest.mark.gpu

EDGE = [1, 2, 63, 64, 65, 127, 128, 129, 191, 200, 257]
FORMS = ["auto", "tc_split", "tc_single", "tc_pipe", "simt"]


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_11_b200 import kda
    return kda


def draw(seed):
    rng = np.random.default_rng(seed)
    form = FORMS[seed % len(FORMS)]
    packed = bool(rng.integers(2))
    H = int(rng.integers(1, 4))
    s0 = float(rng.choice([0.0, 0.1]))
    if packed:
        n = int(rng.integers(2, 6))
        lens = [int(rng.choice(EDGE)) if rng.random() < 0.7 else int(rng.integers(0, 300)) for _ in range(n)]
        if rng.random() < 0.3:
            lens[int(rng.integers(n))] = 0
        return form, True, H, s0, lens
    B = int(rng.integers(1, 3))
    T = int(rng.choice(EDGE)) if rng.random() < 0.5 else int(rng.integers(1, 600))
    return form, False, H, s0, (B, T)


@pytest.mark.parametrize("seed", range(24))
def test_random_case(K, oracle_mod, seed):
    form, packed, H, s0, shape = draw(seed)
    if packed:
        lens = shape
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        inp = case(1, int(cu[-1]), H, 128, 128, "bf16", seed=1000 + seed, s0_std=s0, num_states=len(lens))
        inp["cu_seqlens"] = torch.tensor(cu, device="cuda")
        units = [(n, h) for n in range(len(lens)) for h in range(H)]
        cu_list = [int(x) for x in cu]
    else:
        B, T = shape
        inp = case(B, T, H, 128, 128, "bf16", seed=1000 + seed, s0_std=s0)
        units = [(b, h) for b in range(B) for h in range(H)]
        cu_list = None
    if seed % 3 == 0:  # decays at g_min on a quarter of the channels
        inp["g"][..., :32] = -5.0
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, ST = K.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), chunk=64,
                          cu_seqlens=inp.get("cu_seqlens"), path=form, dev_status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    o_ref, S_ref = oracle_forward(oracle_mod, inp)
    compare_units(o, ST, o_ref, S_ref, units, cu_list, tol=TOL["bf16"], label=f"random {seed} {form}")
