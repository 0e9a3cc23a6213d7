"""The oracle against the figures the pages print (tests/golden/pages_figures.txt)."""
import math
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def figures():
    out = {}
    with open(os.path.join(HERE, "golden", "pages_figures.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                out[k] = float(v)
    return out


def _unit(rng, T, dk, dv):
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -5.0 / (1.0 + np.exp(-rng.standard_normal((T, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    return q, k, v, g, beta


def test_kcp_composition_error_at_machine_precision(oracle_mod):
    """The pages' script finds the KCP composition exact to machine precision
    (max error 6.94e-18 on its own small case) and the 4-rank prefix scan
    exact to 1.39e-17. The oracle's pairs composed over two halves, and
    scanned over 4 ranks, must agree with one sequential pass to within a
    few ulp of the state's magnitude, i.e. the same machine-precision level."""
    fig = figures()
    rng = np.random.default_rng(2024)
    T, dk, dv = 64, 8, 8
    q, k, v, g, beta = _unit(rng, T, dk, dv)
    _, S_seq = oracle_mod.forward(q, k, v, g, beta)
    scale = np.max(np.abs(S_seq))
    # composition of two halves
    Ma, Sa = oracle_mod.segment_pair(q[:32], k[:32], v[:32], g[:32], beta[:32], C=16)
    Mb, Sb = oracle_mod.segment_pair(q[32:], k[32:], v[32:], g[32:], beta[32:], C=16)
    _, S2 = oracle_mod.kcp_compose(Mb, Sb, Ma, Sa)
    err_comp = np.max(np.abs(S2 - S_seq))
    # 4-rank prefix scan
    Ms, Ss = zip(*[oracle_mod.segment_pair(q[a:a + 16], k[a:a + 16], v[a:a + 16], g[a:a + 16],
                                           beta[a:a + 16], C=16) for a in range(0, 64, 16)])
    S_in = oracle_mod.kcp_scan(np.stack(Ms), np.stack(Ss))
    err_scan = np.max(np.abs(S_in[-1] - S_seq))
    eps = np.finfo(np.float64).eps
    # The pages print absolute errors (6.94e-18 for one composition, 1.39e-17 for
    # the 4-rank scan) on a case of unstated size and magnitude; read as "exact up
    # to rounding", they fix the level, not the digits. The oracle's own errors,
    # measured here on a case of its own, must sit at that level: a few ulp of the
    # state's magnitude, and the scan (three compositions in a row) no more than a
    # few times the single composition, as in the pages' pair of figures.
    assert err_comp <= 64 * eps * max(scale, 1.0)
    assert err_scan <= 64 * eps * max(scale, 1.0)
    ratio_pages = fig["kcp_scan_4ranks_max_error"] / fig["kcp_composition_max_error"]
    assert err_scan <= 4 * ratio_pages * max(err_comp, eps * scale)


def test_state_size_figure():
    """About 217 per request: 69 KDA layers x 96 heads x a 128 x 128 state at
    2 bytes per element is 217,055,232 bytes (the figure is in decimal MB, and
    matches a bf16 state; the fp32 state this library keeps is twice that)."""
    fig = figures()
    b = int(fig["kda_layers"] * fig["kda_heads"] * fig["kda_head_dim"] ** 2 * 2)
    assert b == 217_055_232
    assert round(b / 1e6) == fig["kda_state_per_request_mb"]


def test_g_min_subtile_headroom():
    """16 tokens at g_min give a cumulative factor e^80 ~ 5.5e34, inside the
    bf16 range (~3e38); twice that (e^160, the g_min = -10 case) overflows."""
    fig = figures()
    e = math.exp(-fig["subtile_tokens"] * fig["g_min"])
    assert abs(e / fig["exp_16_gmin"] - 1) < 0.01
    bmax = torch.finfo(torch.bfloat16).max
    assert abs(bmax / fig["bf16_max"] - 1) < 0.15
    assert e < bmax and math.exp(160) > bmax
    assert torch.isfinite(torch.tensor(e, dtype=torch.bfloat16))
    assert torch.isfinite(torch.tensor(e, dtype=torch.float32))
