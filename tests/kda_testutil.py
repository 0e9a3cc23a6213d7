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


class UnitErrors(tuple):
    """(e_o, e_s): normwise errors pooled over the compared units, unpacking as
    before; ``worst_o`` / ``worst_s`` and ``worst_unit_o`` / ``worst_unit_s``
    are the largest per-(sequence, head) errors and the units they come from."""

    def __new__(cls, e_o, e_s, worst):
        t = super().__new__(cls, (e_o, e_s))
        t.worst_o, t.worst_unit_o, t.worst_s, t.worst_unit_s = worst
        return t


SHORT_UNIT = 64        # units with fewer output tokens than one chunk
SHORT_UNIT_FACTOR = 3  # ... are gated at this multiple of the bar


def compare_units(o_gpu, ST_gpu, o_ref, ST_ref, units, cu=None, tol=None, label=""):
    """Normwise errors over the given (n, h) units only (o_ref may be a dict
    keyed by unit, as oracle_forward returns for large batches). Pooled errors
    and the worst single unit are both computed; with ``tol`` both are asserted
    to stay below it (a defect confined to a few units cannot hide behind the
    pooled norm), and the worst unit is printed. The output of a unit shorter
    than one chunk is gated at SHORT_UNIT_FACTOR x tol: over a handful of tokens
    one token whose output is a small difference of larger terms (q.k near zero)
    dominates the unit's norm, and its error is set by the bf16 rounding of the
    operands of that dot product, not by the size of the output."""
    if cu is None:
        sel = lambda a, n, h: a[n, :, h]
    else:
        sel = lambda a, n, h: a[0, cu[n]:cu[n + 1], h]
    og, orf, sg, sr = [], [], [], []
    worst = [0.0, None, 0.0, None]
    for n, h in units:
        a = to_f64(sel(o_gpu, n, h)).ravel()
        b = (o_ref[(n, h)] if isinstance(o_ref, dict) else sel(o_ref, n, h)).ravel()
        og.append(a); orf.append(b)
        if b.size and np.linalg.norm(b) > 0:
            e = rel(a, b)
            tokens = len(sel(o_gpu, n, h))
            if tokens < SHORT_UNIT:  # compared against the bar as a multiple of it
                e = e / SHORT_UNIT_FACTOR
            if e > worst[0] or worst[1] is None:
                worst[0], worst[1] = e, (n, h)
        if ST_gpu is not None:
            c, d = to_f64(ST_gpu[n, h]).ravel(), ST_ref[n, h].ravel()
            sg.append(c); sr.append(d)
            e = rel(c, d)
            if e > worst[2] or worst[3] is None:
                worst[2], worst[3] = e, (n, h)
    e_o = rel(np.concatenate(og), np.concatenate(orf))
    e_s = rel(np.concatenate(sg), np.concatenate(sr)) if ST_gpu is not None else None
    res = UnitErrors(e_o, e_s, worst)
    print(f"[parity{' ' + label if label else ''}] units={len(units)} pooled o={e_o:.3e}"
          + (f" S_T={e_s:.3e}" if e_s is not None else "")
          + f" worst o={worst[0]:.3e} (short units / {SHORT_UNIT_FACTOR}) at {worst[1]}"
          + (f" worst S_T={worst[2]:.3e} at {worst[3]}" if ST_gpu is not None else ""))
    if tol is not None:
        assert e_o < tol and res.worst_o < tol, ("o", e_o, res.worst_o, res.worst_unit_o)
        if e_s is not None:
            assert e_s < tol and res.worst_s < tol, ("S_T", e_s, res.worst_s, res.worst_unit_s)
    return res


def parity_streamed(oracle, inp, o_gpu, ST_gpu, units, tol, label="", workers=None):
    """Oracle parity over many (n, h) units without holding their fp64 outputs:
    each unit's inputs are copied to the host, run through the oracle and
    compared in a worker thread (the oracle is a C library called through
    ctypes, which releases the GIL, so the units run on all host cores), and
    only the per-unit error sums are kept. Asserts the pooled and the worst
    per-unit normwise error of o and S_T against ``tol``; returns
    (pooled_o, pooled_S, worst_o, worst_S)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    k = inp["k"]
    B, T, H, dk = k.shape
    cu = inp.get("cu_seqlens")
    cu = None if cu is None else [int(x) for x in cu.cpu().tolist()]
    spans = [(b, 0, T) for b in range(B)] if cu is None else \
        [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    S0 = inp.get("S0")

    def one(unit):
        n, h = unit
        b, t0, t1 = spans[n]
        a = [to_f64(inp[x][b, t0:t1, h]) for x in ("q", "k", "v", "g", "beta")]
        s0 = None if S0 is None else to_f64(S0[n, h])
        ou, su = oracle.forward(*a, S0=s0)
        og = to_f64(o_gpu[b, t0:t1, h])
        sg = to_f64(ST_gpu[n, h])
        return (float(np.sum((og - ou) ** 2)), float(np.sum(ou ** 2)),
                float(np.sum((sg - su) ** 2)), float(np.sum(su ** 2)))

    workers = workers or max(1, min(32, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        sums = list(ex.map(one, units))
    no = sum(x[0] for x in sums); do = sum(x[1] for x in sums)
    ns = sum(x[2] for x in sums); ds = sum(x[3] for x in sums)
    pooled_o = float(np.sqrt(no / do)) if do > 0 else float(np.sqrt(no))
    pooled_s = float(np.sqrt(ns / ds)) if ds > 0 else float(np.sqrt(ns))
    per_o = [(np.sqrt(x[0] / x[1]), u) for x, u in zip(sums, units) if x[1] > 0]
    per_s = [(np.sqrt(x[2] / x[3]) if x[3] > 0 else np.sqrt(x[2]), u) for x, u in zip(sums, units)]
    wo, wu_o = max(per_o) if per_o else (0.0, None)
    ws, wu_s = max(per_s)
    print(f"[parity{' ' + label if label else ''}] units={len(units)} pooled o={pooled_o:.3e} "
          f"S_T={pooled_s:.3e} worst o={wo:.3e} at {wu_o} worst S_T={ws:.3e} at {wu_s}")
    assert pooled_o < tol and wo < tol, ("o", pooled_o, wo, wu_o)
    assert pooled_s < tol and ws < tol, ("S_T", pooled_s, ws, wu_s)
    return pooled_o, pooled_s, wo, ws


def case(B, T, H, dk, dv, dtype, seed, s0_std=0.0, g_min_frac=0.0, device="cuda", num_states=None):
    return make_inputs(B, T, H, dk, dv, dtype, seed=seed, device=device, s0_std=s0_std,
                       g_min_frac=g_min_frac, num_states=num_states)
