"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formula: each compares it with an
independent formulation (dense transition-matrix products, exact rational
arithmetic, closed forms, invariants, the KCP pair algebra) or with a figure
the pages print. Sources: "Exercices" Q7 (the three operations), Q8 (g_min),
Q9 (||k|| = 1), Q21-Q22 (KCP pair and its associativity); "Reproduire Kimi K3"
(the verification script's KCP errors).
"""
from fractions import Fraction

import numpy as np
import pytest

TOL = 1e-14


def rel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return np.linalg.norm(x - ref) / (n if n > 0 else 1.0)


def rand_unit(rng, T, dk, dv, s0=True, gscale=1.0):
    """A random unit with the workloads' distributions (unit-norm q, k)."""
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -5.0 / (1.0 + np.exp(-rng.standard_normal((T, dk)))) * gscale
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = 0.5 * rng.standard_normal((dv, dk)) if s0 else None
    return q, k, v, g, beta, S0


def dense_bruteforce(q, k, v, g, beta, S0):
    """Independent formulation: explicit dense transitions
    M_t = (I - beta_t k_t k_t^T) Diag(exp g_t) and plain matrix products,
    S_T = M_T..M_1 S0 + sum_t M_T..M_{t+1} beta_t k_t v_t^T,  o_t = S_t^T q_t.
    States here are S (dk x dv), not the transposed storage."""
    T, dk = k.shape
    dv = v.shape[1]
    Ms = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]
    S0m = np.zeros((dk, dv)) if S0 is None else S0.T
    o = np.zeros((T, dv))
    for t in range(T):
        # S_t = (M_t ... M_1) S0 + sum_{s<=t} (M_t ... M_{s+1}) beta_s k_s v_s^T
        St = np.zeros((dk, dv))
        P = np.eye(dk)
        for s in range(t, -1, -1):
            St += P @ (beta[s] * np.outer(k[s], v[s]))
            P = P @ Ms[s]
        St += P @ S0m
        o[t] = St.T @ q[t]
    return o, St.T


# --------------------------------------------------------------------- forms

@pytest.mark.parametrize("C", [1, 2, 3, 16, 64, 150])
def test_sequential_equals_chunked(oracle_mod, C):
    rng = np.random.default_rng(11 + C)
    for gscale in (1.0, 0.02):
        q, k, v, g, beta, S0 = rand_unit(rng, 150, 16, 12, gscale=gscale)
        o_s, S_s = oracle_mod.forward(q, k, v, g, beta, S0)
        o_c, S_c = oracle_mod.chunked(q, k, v, g, beta, S0, C=C)
        assert rel(o_c, o_s) < TOL and rel(S_c, S_s) < TOL


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
def test_bruteforce_dense(oracle_mod, T):
    rng = np.random.default_rng(100 + T)
    q, k, v, g, beta, S0 = rand_unit(rng, T, 6, 5)
    o_b, S_b = dense_bruteforce(q, k, v, g, beta, S0)
    o_s, S_s = oracle_mod.forward(q, k, v, g, beta, S0)
    o_c, S_c = oracle_mod.chunked(q, k, v, g, beta, S0, C=3)
    assert rel(o_s, o_b) < 1e-14 and rel(S_s, S_b) < 1e-14
    assert rel(o_c, o_b) < 1e-14 and rel(S_c, S_b) < 1e-14


def test_exact_rational_tiny(oracle_mod):
    """T=3, dk=dv=2 in exact rationals (alpha = 1/2, 1, 1/4 -> g = log alpha).
    The recurrence is applied with Fractions to dense 2x2 matrices."""
    alphas = [[Fraction(1, 2), Fraction(1)], [Fraction(1), Fraction(1, 4)], [Fraction(1, 2), Fraction(1, 2)]]
    ks = [[Fraction(3, 5), Fraction(4, 5)], [Fraction(1), Fraction(0)], [Fraction(0), Fraction(1)]]
    qs = [[Fraction(1), Fraction(0)], [Fraction(3, 5), Fraction(-4, 5)], [Fraction(0), Fraction(1)]]
    vs = [[Fraction(2), Fraction(-1)], [Fraction(1, 2), Fraction(3)], [Fraction(-1), Fraction(1)]]
    betas = [Fraction(1, 2), Fraction(1), Fraction(1, 4)]
    S = [[Fraction(1, 10), Fraction(0)], [Fraction(0), Fraction(-1, 5)]]  # S[i][j], dk x dv
    S0 = [row[:] for row in S]
    outs = []
    for t in range(3):
        a, kk, vv, b, qq = alphas[t], ks[t], vs[t], betas[t], qs[t]
        D = [[a[i] * S[i][j] for j in range(2)] for i in range(2)]
        kTD = [sum(kk[i] * D[i][j] for i in range(2)) for j in range(2)]
        S = [[D[i][j] - b * kk[i] * kTD[j] + b * kk[i] * vv[j] for j in range(2)] for i in range(2)]
        outs.append([sum(S[i][j] * qq[i] for i in range(2)) for j in range(2)])
    f = lambda M: np.array([[float(x) for x in r] for r in M])
    g = np.log(f(alphas))
    o, ST = oracle_mod.forward(f(qs), f(ks), f(vs), g, np.array([float(b) for b in betas]),
                               f(S0).T.copy())
    assert np.max(np.abs(o - f(outs))) < 1e-15
    assert np.max(np.abs(ST - f(S).T)) < 1e-15


# ------------------------------------------------------------------ KCP pair

@pytest.mark.parametrize("gscale", [1.0, 0.02])
@pytest.mark.parametrize("P", [2, 4, 7])
def test_kcp_scan_any_split(oracle_mod, P, gscale):
    """Prefix scan over P segment pairs equals one sequential pass ("Exercices"
    Q22; the pages' 4-rank scan check). The weak-decay case keeps the incoming
    state's contribution large, so an error in any M_p shows."""
    rng = np.random.default_rng(7 * P)
    T, dk, dv = 203, 12, 10
    q, k, v, g, beta, S0 = rand_unit(rng, T, dk, dv, gscale=gscale)
    cuts = np.sort(rng.choice(np.arange(1, T), size=P - 1, replace=False))
    bounds = [0, *cuts.tolist(), T]
    Ms, Ss = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        M, Sl = oracle_mod.segment_pair(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], C=16)
        Ms.append(M); Ss.append(Sl)
    S_in = oracle_mod.kcp_scan(np.stack(Ms), np.stack(Ss), S0)
    o_s, S_s = oracle_mod.forward(q, k, v, g, beta, S0)
    assert rel(S_in[-1], S_s) < TOL
    # replaying each segment from its scanned entry state gives the outputs
    for p, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        o_p, S_p = oracle_mod.forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], S_in[p])
        assert rel(o_p, o_s[a:b]) < TOL
        assert rel(S_p, S_in[p + 1]) < TOL


def test_segment_pair_is_affine_map(oracle_mod):
    """(M, S~) summarises the segment: S_out = M S_in + S~ for any S_in, and
    M is the dense product of the per-token transitions ("Exercices", Q21)."""
    rng = np.random.default_rng(5)
    T, dk, dv = 40, 8, 6
    q, k, v, g, beta, _ = rand_unit(rng, T, dk, dv, s0=False)
    M, Sl = oracle_mod.segment_pair(q, k, v, g, beta, C=16)
    Mdense = np.eye(dk)
    for t in range(T):
        Mdense = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) @ Mdense
    assert rel(M, Mdense) < TOL
    for _ in range(3):
        S_in = rng.standard_normal((dv, dk))
        _, S_out = oracle_mod.forward(q, k, v, g, beta, S_in)
        assert rel(S_out, (M @ S_in.T + Sl.T).T) < TOL


def test_kcp_compose_associative(oracle_mod):
    rng = np.random.default_rng(9)
    dk, dv = 7, 5
    pairs = [(rng.standard_normal((dk, dk)), rng.standard_normal((dv, dk))) for _ in range(3)]
    (M3, S3), (M2, S2), (M1, S1) = pairs[2], pairs[1], pairs[0]
    a = oracle_mod.kcp_compose(*oracle_mod.kcp_compose(M3, S3, M2, S2), M1, S1)
    b = oracle_mod.kcp_compose(M3, S3, *oracle_mod.kcp_compose(M2, S2, M1, S1))
    assert rel(a[0], b[0]) < TOL and rel(a[1], b[1]) < TOL
    # the composition of explicit affine maps: S -> M S + S~
    X = rng.standard_normal((dv, dk))
    step = lambda M, S, X: (M @ X.T + S.T).T
    assert rel(step(*a, X), step(M3, S3, step(M2, S2, step(M1, S1, X)))) < TOL


# -------------------------------------------------------- closed forms

def test_identity_transition(oracle_mod):
    """beta = 0 and g = 0: the transition is I and nothing is written, so
    S_T = S0 exactly and o_t = S0^T q_t."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = rand_unit(rng, 33, 16, 8)
    g[:] = 0.0; beta[:] = 0.0
    for fn in (oracle_mod.forward, lambda *a: oracle_mod.chunked(*a, C=16)):
        o, ST = fn(q, k, v, g, beta, S0)
        assert np.array_equal(ST, S0)
        assert np.max(np.abs(o - q @ S0.T)) < 1e-15


def test_beta_zero_is_pure_decay(oracle_mod):
    """beta = 0: S_T = Diag(exp(sum_t g_t)) S0; with g = g_min = -5 everywhere
    that is exp(-5 T) S0 ("Exercices", Q8)."""
    rng = np.random.default_rng(4)
    q, k, v, g, beta, S0 = rand_unit(rng, 20, 8, 6)
    beta[:] = 0.0
    _, ST = oracle_mod.forward(q, k, v, g, beta, S0)
    assert rel(ST, S0 * np.exp(g.sum(0))[None, :]) < 1e-14
    g[:] = -5.0
    _, ST = oracle_mod.chunked(q, k, v, g, beta, S0, C=8)
    assert rel(ST, S0 * np.exp(-5.0 * 20)) < 1e-14


def test_delta_rule_overwrite(oracle_mod):
    """g = 0, beta = 1, k = e_i: row i of S is replaced by v_t^T (erase what the
    key holds, then write), every other row is unchanged."""
    rng = np.random.default_rng(6)
    dk, dv, T = 5, 4, 6
    S = rng.standard_normal((dk, dv))
    idx = [2, 0, 2, 4, 1, 3]
    q = rng.standard_normal((T, dk)); v = rng.standard_normal((T, dv))
    k = np.zeros((T, dk)); k[np.arange(T), idx] = 1.0
    g = np.zeros((T, dk)); beta = np.ones(T)
    o, ST = oracle_mod.forward(q, k, v, g, beta, S.T.copy())
    Sref = S.copy()
    for t in range(T):
        Sref[idx[t]] = v[t]
        assert np.allclose(o[t], Sref.T @ q[t], rtol=0, atol=1e-14)
    assert np.allclose(ST, Sref.T, rtol=0, atol=1e-15)


# -------------------------------------------------------------- invariants

def test_linear_in_v_and_s0(oracle_mod):
    rng = np.random.default_rng(8)
    q, k, v1, g, beta, S1 = rand_unit(rng, 50, 8, 6)
    v2 = rng.standard_normal(v1.shape); S2 = rng.standard_normal(S1.shape)
    a, b = 0.7, -1.3
    o1, T1 = oracle_mod.chunked(q, k, v1, g, beta, S1, C=16)
    o2, T2 = oracle_mod.chunked(q, k, v2, g, beta, S2, C=16)
    o3, T3 = oracle_mod.chunked(q, k, a * v1 + b * v2, g, beta, a * S1 + b * S2, C=16)
    assert rel(o3, a * o1 + b * o2) < TOL and rel(T3, a * T1 + b * T2) < TOL


def test_dv_columns_separable(oracle_mod):
    """The recurrence acts on S from the left only, so the dv columns evolve
    independently: running two halves of v equals running all of it."""
    rng = np.random.default_rng(10)
    q, k, v, g, beta, S0 = rand_unit(rng, 70, 8, 10)
    o, ST = oracle_mod.forward(q, k, v, g, beta, S0)
    oa, Ta = oracle_mod.chunked(q, k, v[:, :4], g, beta, S0[:4], C=16)
    ob, Tb = oracle_mod.chunked(q, k, v[:, 4:], g, beta, S0[4:], C=16)
    assert rel(np.concatenate([oa, ob], 1), o) < TOL
    assert rel(np.concatenate([Ta, Tb], 0), ST) < TOL


def test_contraction_bound(oracle_mod):
    """||k|| = 1, g <= 0, beta in [0, 1] make (I - beta k k^T) Diag(alpha) a
    contraction ("Exercices", Q9), so ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||_2."""
    rng = np.random.default_rng(12)
    q, k, v, g, beta, S0 = rand_unit(rng, 60, 8, 6, gscale=0.05)
    S = S0.copy()
    for t in range(60):
        prev = np.linalg.norm(S, 2)
        oracle_mod.decode_step(q[t], k[t], v[t], g[t], beta[t], S)
        assert np.linalg.norm(S, 2) <= prev + beta[t] * np.linalg.norm(v[t]) + 1e-12


def test_chaining_equals_one_pass(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v, g, beta, S0 = rand_unit(rng, 97, 8, 8)
    o, ST = oracle_mod.chunked(q, k, v, g, beta, S0, C=16)
    o1, Sm = oracle_mod.chunked(q[:41], k[:41], v[:41], g[:41], beta[:41], S0, C=16)
    o2, S2 = oracle_mod.chunked(q[41:], k[41:], v[41:], g[41:], beta[41:], Sm, C=16)
    assert rel(np.concatenate([o1, o2]), o) < TOL and rel(S2, ST) < TOL


def test_decode_steps_equal_forward(oracle_mod):
    rng = np.random.default_rng(14)
    q, k, v, g, beta, S0 = rand_unit(rng, 9, 8, 8)
    o, ST = oracle_mod.forward(q, k, v, g, beta, S0)
    S = S0.copy()
    for t in range(9):
        ot = oracle_mod.decode_step(q[t], k[t], v[t], g[t], beta[t], S)
        assert rel(ot, o[t]) < 1e-15
    assert rel(S, ST) < 1e-15


def test_g_min_runs_stay_finite(oracle_mod):
    """Whole channels at g = g_min = -5 over >= 64 tokens: the chunked form's
    pairwise exponents stay in range and it still equals the sequential one."""
    rng = np.random.default_rng(15)
    q, k, v, g, beta, S0 = rand_unit(rng, 130, 16, 8)
    g[:, ::2] = -5.0
    o_s, S_s = oracle_mod.forward(q, k, v, g, beta, S0)
    o_c, S_c = oracle_mod.chunked(q, k, v, g, beta, S0, C=64)
    assert np.all(np.isfinite(o_c)) and rel(o_c, o_s) < TOL and rel(S_c, S_s) < TOL


def test_forward_tokens_layout(oracle_mod):
    """The token-major batch driver slices units the way the library lays them
    out ([B,T,H,d], states [N,H,dv,dk], varlen offsets)."""
    rng = np.random.default_rng(16)
    T, H, dk, dv = 30, 3, 4, 5
    # build a [1, T, H, *] batch from H independent units
    units = [rand_unit(rng, T, dk, dv) for _ in range(H)]
    q = np.stack([u[0] for u in units], 1)[None]
    k = np.stack([u[1] for u in units], 1)[None]
    v = np.stack([u[2] for u in units], 1)[None]
    g = np.stack([u[3] for u in units], 1)[None]
    beta = np.stack([u[4] for u in units], 1)[None]
    cu = [0, 11, 30]
    S0 = rng.standard_normal((2, H, dv, dk))
    o, ST = oracle_mod.forward_tokens(q, k, v, g, beta, S0, cu_seqlens=cu)
    for n, (a, b) in enumerate([(0, 11), (11, 30)]):
        for h in range(H):
            ou, su = oracle_mod.forward(q[0, a:b, h], k[0, a:b, h], v[0, a:b, h], g[0, a:b, h],
                                        beta[0, a:b, h], S0[n, h])
            assert np.array_equal(o[0, a:b, h], ou) and np.array_equal(ST[n, h], su)
