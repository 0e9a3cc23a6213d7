"""Python bindings of the fp64 KDA oracle (``oracle/kda_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module; the product package never
does, and the two share no code. Every function here is argument marshalling
around the C oracle (numpy float64 arrays in, numpy float64 arrays out), plus a
loop over (sequence, head) units for the token-major ``[B, T, H, d]`` layouts;
no arithmetic of the method lives in Python.

Per-unit layouts (row-major): q, k, g ``[T, dk]``; v, o ``[T, dv]``; beta
``[T]``; states ``[dv, dk]`` (element (i, j) of S at ``[j, i]``); the KCP
transition M ``[dk, dk]``.

Parity pins: see ``tests/test_oracle_*.py`` (sequential vs chunked vs KCP scan,
dense brute force, closed forms, invariants and the pages' printed figures).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_SO = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp64, no fast-math) if it is stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def load(path: str):
    """Load a compiled oracle library and declare its signatures."""
    L = ctypes.CDLL(path)
    i, d = ctypes.c_int, ctypes.c_double
    L.kda_oracle_forward.argtypes = [i, i, i, _D, _D, _D, _D, _D, _D, _D, _D]
    L.kda_oracle_chunked.argtypes = [i, i, i, i, _D, _D, _D, _D, _D, _D, _D, _D]
    L.kda_oracle_decode_step.argtypes = [i, i, _D, _D, _D, _D, d, _D, _D]
    L.kda_oracle_kcp_compose.argtypes = [i, i, _D, _D, _D, _D, _D, _D]
    L.kda_oracle_segment_pair.argtypes = [i, i, i, i, _D, _D, _D, _D, _D, _D, _D]
    L.kda_oracle_kcp_scan.argtypes = [i, i, i, _D, _D, _D, _D]
    for f in ("kda_oracle_forward", "kda_oracle_chunked", "kda_oracle_decode_step",
              "kda_oracle_kcp_compose", "kda_oracle_segment_pair", "kda_oracle_kcp_scan"):
        getattr(L, f).restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _c(a):
    """C-contiguous float64 copy/view of ``a`` (None stays None)."""
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(_D)


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed (rc={rc})")


def _unit_args(q, k, v, g, beta):
    q, k, v, g, beta = (_c(x) for x in (q, k, v, g, beta))
    T, dk = k.shape
    dv = v.shape[1]
    assert q.shape == (T, dk) and g.shape == (T, dk) and v.shape == (T, dv) and beta.shape == (T,)
    return q, k, v, g, beta, T, dk, dv


def forward(q, k, v, g, beta, S0=None):
    """Sequential recurrence for one unit. Returns (o [T, dv], S_T [dv, dk])."""
    q, k, v, g, beta, T, dk, dv = _unit_args(q, k, v, g, beta)
    S0 = _c(S0)
    o = np.empty((T, dv)); ST = np.empty((dv, dk))
    _check(lib().kda_oracle_forward(T, dk, dv, _p(q), _p(k), _p(v), _p(g), _p(beta),
                                    _p(S0), _p(o), _p(ST)), "kda_oracle_forward")
    return o, ST


def chunked(q, k, v, g, beta, S0=None, C=64):
    """Chunked (UT/KCP) form for one unit, chunks of C tokens. Returns (o, S_T)."""
    q, k, v, g, beta, T, dk, dv = _unit_args(q, k, v, g, beta)
    S0 = _c(S0)
    o = np.empty((T, dv)); ST = np.empty((dv, dk))
    _check(lib().kda_oracle_chunked(T, dk, dv, int(C), _p(q), _p(k), _p(v), _p(g), _p(beta),
                                    _p(S0), _p(o), _p(ST)), "kda_oracle_chunked")
    return o, ST


def decode_step(q, k, v, g, beta, St):
    """One-token step for one unit; ``St`` ([dv, dk] float64, C-contiguous) is
    updated in place. Returns o [dv]."""
    assert isinstance(St, np.ndarray) and St.dtype == np.float64 and St.flags.c_contiguous
    q, k, v, g = (_c(x) for x in (q, k, v, g))
    dk, dv = k.shape[0], v.shape[0]
    o = np.empty(dv)
    _check(lib().kda_oracle_decode_step(dk, dv, _p(q), _p(k), _p(v), _p(g), float(beta),
                                        _p(St), _p(o)), "kda_oracle_decode_step")
    return o


def kcp_compose(M2, S2, M1, S1):
    """(M2, S~2) o (M1, S~1) = (M2 M1, M2 S~1 + S~2)."""
    M2, S2, M1, S1 = (_c(x) for x in (M2, S2, M1, S1))
    dk, dv = M2.shape[0], S2.shape[0]
    Mo = np.empty((dk, dk)); So = np.empty((dv, dk))
    _check(lib().kda_oracle_kcp_compose(dk, dv, _p(M2), _p(S2), _p(M1), _p(S1), _p(Mo), _p(So)),
           "kda_oracle_kcp_compose")
    return Mo, So


def segment_pair(q, k, v, g, beta, C=64):
    """KCP pair (M [dk, dk], S~ [dv, dk]) of one segment (chunk pairs composed)."""
    q, k, v, g, beta, T, dk, dv = _unit_args(q, k, v, g, beta)
    M = np.empty((dk, dk)); S = np.empty((dv, dk))
    _check(lib().kda_oracle_segment_pair(T, dk, dv, int(C), _p(q), _p(k), _p(v), _p(g), _p(beta),
                                         _p(M), _p(S)), "kda_oracle_segment_pair")
    return M, S


def kcp_scan(Ms, Ss, S0=None):
    """Exclusive prefix scan of segment pairs. Returns S_in [P+1, dv, dk]."""
    Ms, Ss, S0 = _c(Ms), _c(Ss), _c(S0)
    P, dk = Ms.shape[0], Ms.shape[1]
    dv = Ss.shape[1]
    out = np.empty((P + 1, dv, dk))
    _check(lib().kda_oracle_kcp_scan(P, dk, dv, _p(Ms), _p(Ss), _p(S0), _p(out)),
           "kda_oracle_kcp_scan")
    return out


def forward_tokens(q, k, v, g, beta, S0=None, cu_seqlens=None, units=None, chunk=None):
    """Loop the unit oracle over a token-major batch.

    q, k, g ``[B, T, H, dk]``; v ``[B, T, H, dv]``; beta ``[B, T, H]`` (numpy or
    anything ``np.asarray`` accepts). With ``cu_seqlens`` (int offsets,
    ``[N+1]``), B must be 1 and sequence n is tokens ``cu[n]:cu[n+1]``.
    ``S0`` is ``[N, H, dv, dk]`` (N = B or the number of sequences) or None.
    ``units`` optionally restricts the work to a list of (n, h) pairs.
    ``chunk`` selects the chunked form instead of the sequential one.

    Returns ``(o, S_T)`` with o like v (NaN where a unit was not computed) and
    S_T ``[N, H, dv, dk]`` (NaN for units not computed).
    """
    q, k, v, g, beta = (np.asarray(x) for x in (q, k, v, g, beta))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in np.asarray(cu_seqlens).tolist()]
        assert B == 1
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    N = len(spans)
    o = np.full((B, T, H, dv), np.nan)
    ST = np.full((N, H, dv, dk), np.nan)
    todo = units if units is not None else [(n, h) for n in range(N) for h in range(H)]
    for n, h in todo:
        b, t0, t1 = spans[n]
        args = (q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h], g[b, t0:t1, h], beta[b, t0:t1, h])
        s0 = None if S0 is None else np.asarray(S0)[n, h]
        if chunk is None:
            ou, su = forward(*args, S0=s0)
        else:
            ou, su = chunked(*args, S0=s0, C=chunk)
        o[b, t0:t1, h] = ou
        ST[n, h] = su
    return o, ST
