"""Seeded synthetic inputs for the KDA recurrence (shared by tests and bench).

This module holds no arithmetic of the method: it only draws random tensors
with the distributions the workloads use and casts them to the storage dtype.
Both the CUDA path and the fp64 oracle are fed from here (the oracle gets the
identical rounded values, widened to float64).

Recipe (one (token, head) row at a time):
  q, k ~ N(0, 1), then divided by their L2 norm over the head dimension
        (the kernel's precondition: "Exercices", Q9 — I - beta k k^T is only
        well conditioned for ||k||_2 = 1; q is normalised the same way);
  v    ~ N(0, 1);
  beta = sigmoid(N(0, 1))                       per (token, head);
  g    = -5 * sigmoid(N(0, 1))                  per element, i.e. inside the
        bounded range [g_min, 0] with g_min = -5 ("Exercices", Q8);
        optionally a fraction of the elements set to exactly g_min;
  S0   ~ N(0, std) fp32, or absent (zero state).
All draws are made in fp32 from one ``torch.Generator`` per tensor, seeded
from (seed, tensor index), then cast to the storage dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

G_MIN = -5.0


@dataclass(frozen=True)
class Workload:
    """A named KDA workload: shapes, dtypes and input distributions."""
    name: str
    H: int
    dk: int
    dv: int
    dtype: str                      # "f32" or "bf16": storage/compute dtype of q,k,v,g,beta,o
    chunk: int
    B: int = 1
    T: int = 0                      # tokens per sequence (dense batches)
    seqlens: tuple = ()             # packed variable-length sequences (B must be 1)
    s0_std: float = 0.0             # 0 -> no initial state (zeros)
    g_min_frac: float = 0.0         # fraction of g elements set to exactly g_min
    decode_steps: int = 0           # >0: a decode workload (T = 1 per step)
    seg_len: int = 0                # >0: run segment-parallel (segments of seg_len tokens)
    seed: int = 1000
    notes: str = ""

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens) if self.seqlens else self.B

    @property
    def total_tokens(self) -> int:
        return sum(self.seqlens) if self.seqlens else self.B * self.T

    def cu_seqlens(self):
        if not self.seqlens:
            return None
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + n)
        return cu


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> tuple:
    """n lengths drawn log-uniform in [lo, hi] (exp of a uniform in [ln lo, ln hi]),
    rounded to the nearest integer, from a seeded generator."""
    gen = torch.Generator().manual_seed(seed)
    u = torch.rand(n, generator=gen, dtype=torch.float64)
    ls = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    return tuple(int(round(float(x))) for x in ls)


# The workloads of the hot path, named by what they are.
WORKLOADS = {
    "small_f32_T256_d32": Workload(
        name="small_f32_T256_d32", B=1, H=1, T=256, dk=32, dv=32, dtype="f32", chunk=16,
        seed=1000, notes="fp32 parity case"),
    "b2_h4_T2048_d128_bf16": Workload(
        name="b2_h4_T2048_d128_bf16", B=2, H=4, T=2048, dk=128, dv=128, dtype="bf16",
        chunk=64, s0_std=0.02, seed=1001, notes="bf16 parity case with an initial state"),
    "prefill_h96_T8192_d128_bf16": Workload(
        name="prefill_h96_T8192_d128_bf16", B=1, H=96, T=8192, dk=128, dv=128, dtype="bf16",
        chunk=64, g_min_frac=0.10, seed=1002,
        notes="layer shape kda_H=96, kda_hd=128; 10% of g at exactly g_min"),
    "varlen_h96_8seq_d128_bf16": Workload(
        name="varlen_h96_8seq_d128_bf16", B=1, H=96, dk=128, dv=128, dtype="bf16", chunk=64,
        seqlens=varlen_lengths(8, 4096, 131072, seed=1003), seed=1003,
        notes="8 packed sequences, log-uniform lengths in [4096, 131072]"),
    "long_h8_T65536_d128_bf16": Workload(
        name="long_h8_T65536_d128_bf16", B=1, H=8, T=65536, dk=128, dv=128, dtype="bf16",
        chunk=64, g_min_frac=0.10, seg_len=3648, seed=1005,
        notes="one long sequence with few heads (8 units on a 148-SM GPU): segment-parallel, "
              "18 segments of 57 chunks (the last 55), 144 (segment, head) units"),
    "decode_n256_h96_d128": Workload(
        name="decode_n256_h96_d128", B=256, H=96, T=1, dk=128, dv=128, dtype="bf16",
        chunk=64, s0_std=0.02, decode_steps=1000, seed=1004,
        notes="256 requests x 96 heads, fp32 states updated in place"),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(device, seed: int, idx: int) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 1009 + idx)
    return gen


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16", *,
                seed: int = 0, device="cpu", s0_std: float = 0.0, g_min_frac: float = 0.0,
                num_states: int | None = None) -> dict:
    """Draw one batch of inputs.

    Returns a dict with q, k, g ``[B, T, H, dk]``; v ``[B, T, H, dv]``;
    beta ``[B, T, H]`` (all of ``dtype``) and S0 ``[N, H, dv, dk]`` fp32 or None
    (N = ``num_states`` or B). Large tensors are drawn slice by slice along T so
    that the fp32 temporaries stay small.
    """
    tdt = TORCH_DTYPE[dtype]
    out = {}
    step = max(1, (1 << 24) // max(1, B * H * max(dk, dv)))
    specs = [("q", dk, 0), ("k", dk, 1), ("v", dv, 2), ("g", dk, 3)]
    for name, d, idx in specs:
        gen = _gen(device, seed, idx)
        t = torch.empty((B, T, H, d), dtype=tdt, device=device)
        for t0 in range(0, T, step):
            t1 = min(T, t0 + step)
            x = torch.randn((B, t1 - t0, H, d), generator=gen, device=device, dtype=torch.float32)
            if name in ("q", "k"):
                x = _unit_rows(x)
            elif name == "g":
                x = G_MIN * torch.sigmoid(x)
                if g_min_frac > 0:
                    m = torch.rand(x.shape, generator=gen, device=device) < g_min_frac
                    x = torch.where(m, torch.full_like(x, G_MIN), x)
            t[:, t0:t1] = x.to(tdt)
        out[name] = t
    gen = _gen(device, seed, 4)
    out["beta"] = torch.sigmoid(torch.randn((B, T, H), generator=gen, device=device,
                                            dtype=torch.float32)).to(tdt)
    N = B if num_states is None else num_states
    if s0_std > 0:
        gen = _gen(device, seed, 5)
        out["S0"] = s0_std * torch.randn((N, H, dv, dk), generator=gen, device=device,
                                         dtype=torch.float32)
    else:
        out["S0"] = None
    return out


def workload_inputs(w: Workload, device="cpu", step: int | None = None) -> dict:
    """Inputs of a named workload (decode: the inputs of decode step ``step``;
    the initial states are drawn when ``step`` is None or 0)."""
    if w.decode_steps:
        s = 0 if step is None else int(step)
        d = make_inputs(w.B, 1, w.H, w.dk, w.dv, w.dtype, seed=w.seed * 1_000_000 + s,
                        device=device, s0_std=(w.s0_std if s == 0 else 0.0))
        if s != 0:
            d.pop("S0")
        return d
    if w.seqlens:
        d = make_inputs(1, w.total_tokens, w.H, w.dk, w.dv, w.dtype, seed=w.seed, device=device,
                        s0_std=w.s0_std, g_min_frac=w.g_min_frac, num_states=w.num_seqs)
        d["cu_seqlens"] = torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=device)
        return d
    return make_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, seed=w.seed, device=device,
                       s0_std=w.s0_std, g_min_frac=w.g_min_frac)


def to_f64(x):
    """numpy float64 copy of a tensor (exact widening of bf16/fp32 values)."""
    if x is None:
        return None
    return x.detach().to("cpu", torch.float64).numpy()
