"""Helpers shared by the GPU parity tests: run the library and the oracle on
the same seeded inputs and compare normwise."""
import numpy as np
import torch

from linear_attention_recurrence_11_b200.inputs import make_inputs, to_f64

# Tolerances on the normwise relative error ||x - x*||_F / ||x*||_F, per output
# tensor, against the fp64 oracle fed the identical (rounded) inputs.
TOL = {"f32": 1e-4, "bf16": 1e-2}


def rel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def oracle_forward(oracle, inp, units=None, chunk=None):
    """Oracle outputs for the given (n, h) units (default: all), sliced from the
    device inputs unit by unit so that only those units are copied to the host.
    Returns (o, S_T) shaped like the library's outputs, NaN elsewhere."""
    k = inp["k"]
    B, T, H, dk = k.shape
    dv = inp["v"].shape[-1]
    cu = inp.get("cu_seqlens")
    cu = None if cu is None else [int(x) for x in cu.cpu().tolist()]
    spans = [(b, 0, T) for b in range(B)] if cu is None else \
        [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    N = len(spans)
    if units is None:
        units = [(n, h) for n in range(N) for h in range(H)]
    o = np.full((B, T, H, dv), np.nan) if B * T * H * dv <= (1 << 26) else {}
    ST = np.full((N, H, dv, dk), np.nan)
    S0 = inp.get("S0")
    for n, h in units:
        b, t0, t1 = spans[n]
        a = [to_f64(inp[x][b, t0:t1, h]) for x in ("q", "k", "v", "g", "beta")]
        s0 = None if S0 is None else to_f64(S0[n, h])
        if chunk is None:
            ou, su = oracle.forward(*a, S0=s0)
        else:
            ou, su = oracle.chunked(*a, S0=s0, C=chunk)
        if isinstance(o, dict):
            o[(n, h)] = ou
        else:
            o[b, t0:t1, h] = ou
        ST[n, h] = su
    return o, ST


def compare_units(o_gpu, ST_gpu, o_ref, ST_ref, units, cu=None):
    """Normwise errors over the given (n, h) units only (o_ref may be a dict
    keyed by unit, as oracle_forward returns for large batches)."""
    if cu is None:
        sel = lambda a, n, h: a[n, :, h]
    else:
        sel = lambda a, n, h: a[0, cu[n]:cu[n + 1], h]
    og = np.concatenate([to_f64(sel(o_gpu, n, h)).ravel() for n, h in units])
    if isinstance(o_ref, dict):
        orf = np.concatenate([o_ref[(n, h)].ravel() for n, h in units])
    else:
        orf = np.concatenate([sel(o_ref, n, h).ravel() for n, h in units])
    e_o = rel(og, orf)
    e_s = None
    if ST_gpu is not None:
        sg = np.concatenate([to_f64(ST_gpu[n, h]).ravel() for n, h in units])
        sr = np.concatenate([ST_ref[n, h].ravel() for n, h in units])
        e_s = rel(sg, sr)
    return e_o, e_s


def case(B, T, H, dk, dv, dtype, seed, s0_std=0.0, g_min_frac=0.0, device="cuda", num_states=None):
    return make_inputs(B, T, H, dk, dv, dtype, seed=seed, device=device, s0_std=s0_std,
                       g_min_frac=g_min_frac, num_states=num_states)
