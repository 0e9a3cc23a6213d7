"""Plant plausible mistakes in a copy of the oracle source (never in the
oracle itself) and check that the pins catch every one of them.

Each mutant is compiled to a temporary library, swapped in for the real one,
and run through pin checks; a mutant that passes all of them would mean a
pin is missing."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

from test_oracle_pins import dense_bruteforce, rand_unit, rel

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    # sequential recurrence
    "drop_decay": ("ST(S, i, j, dk) *= alpha[i];", ";"),
    "erase_sign": ("const double u = bt * (vt[j] - s);", "const double u = bt * (vt[j] + s);"),
    "write_without_beta": ("const double u = bt * (vt[j] - s);", "const double u = vt[j] - bt * s;"),
    "output_from_key": ("acc += ST(S, i, j, dk) * qt[i];", "acc += ST(S, i, j, dk) * kt[i];"),
    # chunked form
    "gram_transposed": ("c->A[(size_t)r * L + s] * c->W[(size_t)s * dk + i]",
                        "c->A[(size_t)s * L + r] * c->W[(size_t)s * dk + i]"),
    "gram_wrong_exponent": ("const double e = exp(c->G[(size_t)r * dk + i] - c->G[(size_t)s * dk + i]);",
                            "const double e = exp(c->G[(size_t)s * dk + i] - c->G[(size_t)r * dk + i]);"),
    "P_without_diagonal": ("for (int s = 0; s <= r; ++s) acc += c->P",
                           "for (int s = 0; s < r; ++s) acc += c->P"),
    "Kh_missing_decay": ("exp(c->G[(size_t)(L - 1) * dk + i] - c->G[(size_t)r * dk + i]) * k[(size_t)r * dk + i];",
                         "k[(size_t)r * dk + i];"),
    "W_missing_beta": ("double w = beta[r] * exp(", "double w = 1.0 * exp("),
    "U_not_minus_WS": ("U[(size_t)r * dv + j] = c->Ut[(size_t)r * dv + j] - ws;",
                       "U[(size_t)r * dv + j] = c->Ut[(size_t)r * dv + j] + ws;"),
    # KCP composition / scan
    "compose_order": ("acc += M2[(size_t)a * dk + c] * M1[(size_t)c * dk + b];",
                      "acc += M1[(size_t)a * dk + c] * M2[(size_t)c * dk + b];"),
    "compose_drop_local": ("double acc = ST(S2, a, j, dk);", "double acc = 0.0;"),
    "scan_transposed_M": ("acc += Mp[(size_t)a * dk + c] * ST(Sprev, c, j, dk);",
                          "acc += Mp[(size_t)c * dk + a] * ST(Sprev, c, j, dk);"),
}


def _pins_hold() -> bool:
    """A compact run of the pins; False as soon as one fails."""
    rng = np.random.default_rng(77)
    q, k, v, g, beta, S0 = rand_unit(rng, 6, 5, 4)
    o_b, S_b = dense_bruteforce(q, k, v, g, beta, S0)
    o_s, S_s = oracle.forward(q, k, v, g, beta, S0)
    if not (rel(o_s, o_b) < 1e-13 and rel(S_s, S_b) < 1e-13):
        return False
    o_c, S_c = oracle.chunked(q, k, v, g, beta, S0, C=4)
    if not (rel(o_c, o_b) < 1e-13 and rel(S_c, S_b) < 1e-13):
        return False
    # weak decay so that the transitions M (and any error in them) stay visible
    q, k, v, g, beta, S0 = rand_unit(rng, 50, 6, 4, gscale=0.02)
    o_s, S_s = oracle.forward(q, k, v, g, beta, S0)
    bounds = [0, 13, 29, 50]
    pairs = [oracle.segment_pair(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], C=8)
             for a, b in zip(bounds[:-1], bounds[1:])]
    S_in = oracle.kcp_scan(np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs]), S0)
    if not rel(S_in[-1], S_s) < 1e-13:
        return False
    M2, S2 = pairs[1]; M1, S1 = pairs[0]
    Mc, Sc = oracle.kcp_compose(M2, S2, M1, S1)
    _, S_mid = oracle.forward(q[:29], k[:29], v[:29], g[:29], beta[:29], None)
    if not rel(Sc, S_mid) < 1e-13:
        return False
    Md = np.eye(6)
    for t in range(29):
        Md = (np.eye(6) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) @ Md
    return bool(rel(Mc, Md) < 1e-13)


def test_real_oracle_passes():
    assert _pins_hold()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new, 1))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", str(so), str(mut), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(so)))
    assert not _pins_hold(), f"mutant {name} passed every pin"
