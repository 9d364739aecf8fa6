"""Seeded synthetic inputs for MSA decode: shared by the CUDA path and the CPU oracle.

This module generates *inputs only*: fp32 N(0,1) key/value/index-key tensors,
bf16 queries, ragged sequence lengths and "needle" blocks.  It holds none of
the method's arithmetic (no NVFP4 coding, no scoring, no selection, no
attention); both the GPU path and the oracle quantise and process what it
returns on their own.

Every value is a pure function of (seed, tensor id, row, column) — a
counter-based generator — so any sub-range (one sequence, a few blocks) can be
regenerated on its own, and the same code gives bit-identical values on the CPU
and on a CUDA device:

* hashing: the 32-bit ``lowbias32`` integer finalizer from C. Wellons'
  "hash-prospector" (x ^= x>>16; x *= 0x7feb352d; x ^= x>>15;
  x *= 0x846ca68b; x ^= x>>16), evaluated in int64 with the 32x32-bit
  products split into 16-bit halves so nothing overflows;
* normal variates: Box-Muller, sqrt(-2 ln u1) * cos(2 pi u2), evaluated in
  float64 with only IEEE-exact operations (+, -, *, /, sqrt) — ln via frexp
  and the atanh series, cos/sin via quadrant reduction and fixed-length Taylor
  series — then rounded once to float32.  Eager torch runs each of these as a
  separately rounded elementwise op on either device, hence identical bits.

The MiniMax pages (vLLM day-0 support for MiniMax-M3.1-Flash, "A model built
for efficient inference") describe the KV cache as NVFP4 data; the workloads
here are synthetic N(0,1) tensors of the pages' shapes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

MASK32 = 0xFFFFFFFF
MSA_BLOCK = 128  # tokens per MSA block (pages: "blocks of 128 tokens")

# tensor ids of the counter-based streams
TID_K, TID_V, TID_IK, TID_Q, TID_QI, TID_W, TID_LEN, TID_NEEDLE = range(1, 9)


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2**32 for int64 tensors holding uint32 values."""
    lo = x & 0xFFFF
    hi = x >> 16
    return (lo * c + ((hi * (c & 0xFFFF)) << 16)) & MASK32


def lowbias32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def lowbias32_int(x: int) -> int:
    """Scalar version of :func:`lowbias32` on Python ints."""
    x &= MASK32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & MASK32
    x ^= x >> 15
    x = (x * 0x846CA68B) & MASK32
    x ^= x >> 16
    return x


def _stream_key(seed: int, tid: int, stream: int) -> int:
    return lowbias32_int((seed * 0x9E3779B9 + tid * 0x85EBCA6B + stream * 0xC2B2AE35 + 0x27D4EB2F) & MASK32)


def hash_u32(seed: int, tid: int, stream: int, rows: torch.Tensor, cols: torch.Tensor) -> torch.Tensor:
    """32-bit hash of (seed, tid, stream, row, col); rows [R,1] and cols [1,C] int64 (< 2**32)."""
    k = _stream_key(seed, tid, stream)
    r = lowbias32(rows ^ k)
    return lowbias32(lowbias32(cols ^ r) ^ k)


# Fixed-length series coefficients, computed once in Python (identical on every device).
_LN2 = math.log(2.0)
_ATANH_TERMS = [1.0 / (2 * i + 1) for i in range(12)]          # ln m = 2 * sum z^(2i+1)/(2i+1)
_COS_TERMS = [(-1.0) ** i / math.factorial(2 * i) for i in range(12)]
_SIN_TERMS = [(-1.0) ** i / math.factorial(2 * i + 1) for i in range(12)]
_HALF_PI = math.pi / 2.0
_SQRT_HALF = math.sqrt(0.5)


def _horner(t: torch.Tensor, coeffs: Sequence[float]) -> torch.Tensor:
    acc = torch.full_like(t, coeffs[-1])
    for c in reversed(coeffs[:-1]):
        acc = acc * t
        acc = acc + c
    return acc


def _ln_u32p1(h: torch.Tensor) -> torch.Tensor:
    """ln((h + 1) / 2**32) in float64 for int64 h in [0, 2**32)."""
    x = (h + 1).to(torch.float64)
    m, e = torch.frexp(x)  # x = m * 2**e, m in [0.5, 1)
    e = e.to(torch.float64)
    small = m < _SQRT_HALF
    m = torch.where(small, m * 2.0, m)
    e = torch.where(small, e - 1.0, e)
    z = (m - 1.0) / (m + 1.0)
    lnm = _horner(z * z, _ATANH_TERMS) * z * 2.0
    return lnm + (e - 32.0) * _LN2


def _cos_2pi_u32(h: torch.Tensor) -> torch.Tensor:
    """cos(2*pi*h/2**32) in float64 for int64 h in [0, 2**32)."""
    quad = h >> 30
    a = (h & ((1 << 30) - 1)).to(torch.float64) * (2.0 ** -30) * _HALF_PI
    t = a * a
    c = _horner(t, _COS_TERMS)
    s = _horner(t, _SIN_TERMS) * a
    return torch.where(quad == 0, c, torch.where(quad == 1, -s, torch.where(quad == 2, -c, s)))


def normal_block(seed: int, tid: int, rows: torch.Tensor, cols: torch.Tensor) -> torch.Tensor:
    """float32 N(0,1) values at (rows x cols) of stream ``tid``; rows [R,1], cols [1,C] int64."""
    h1 = hash_u32(seed, tid, 0, rows, cols)
    h2 = hash_u32(seed, tid, 1, rows, cols)
    r = torch.sqrt(_ln_u32p1(h1) * -2.0)
    return (r * _cos_2pi_u32(h2)).to(torch.float32)


def normal_tensor(seed: int, tid: int, n_rows: int, n_cols: int, device="cpu",
                  row0: int = 0, col0: int = 0, chunk: int = 1 << 22) -> torch.Tensor:
    """[n_rows, n_cols] float32 N(0,1) with global coordinates (row0+i, col0+j)."""
    out = torch.empty(n_rows, n_cols, dtype=torch.float32, device=device)
    if n_rows == 0 or n_cols == 0:
        return out
    cols = torch.arange(col0, col0 + n_cols, dtype=torch.int64, device=device).view(1, -1)
    rows_per = max(1, chunk // n_cols)
    for i in range(0, n_rows, rows_per):
        j = min(n_rows, i + rows_per)
        rows = torch.arange(row0 + i, row0 + j, dtype=torch.int64, device=device).view(-1, 1)
        out[i:j] = normal_block(seed, tid, rows, cols)
    return out


def uniform_int(seed: int, tid: int, index: int, lo: int, hi: int) -> int:
    """Integer in [lo, hi] from the hash of (seed, tid, index) (CPU, scalar)."""
    h = hash_u32(seed, tid, 2, torch.tensor([[index]]), torch.tensor([[0]])).item()
    return lo + (h * (hi - lo + 1)) // (1 << 32)


# ---------------------------------------------------------------------------
# Workload description and input construction
# ---------------------------------------------------------------------------

@dataclass
class Workload:
    """One synthetic MSA workload (shapes follow the notation B, Tq, Hq, Hkv, D, HI, DI)."""
    name: str
    B: int
    Tq: int
    Hq: int
    Hkv: int
    D: int
    HI: int
    DI: int
    seq_len: int = 0                 # fixed L (includes the Tq query tokens)
    seq_len_range: Optional[tuple] = None  # ragged: L ~ U_int[lo, hi], resampled while L % 128 == 0
    lmax: int = 0
    needles: int = 0
    seed: int = 1234
    weights: bool = False            # indexer head weights w (else NULL = all ones)
    # calibrated per-tensor NVFP4 amax for K, V and index-K: N(0,1) data from the
    # Box-Muller generator is bounded by sqrt(64 ln 2) = 6.66, needles add 0.5*|qbar|
    amax_cal: float = 7.0

    def __post_init__(self):
        if self.lmax == 0:
            self.lmax = self.seq_len_range[1] if self.seq_len_range else self.seq_len

    @property
    def nbmax(self) -> int:
        return (self.lmax + MSA_BLOCK - 1) // MSA_BLOCK


def seq_lens_for(w: Workload) -> List[int]:
    if w.seq_len_range is None:
        return [w.seq_len] * w.B
    lo, hi = w.seq_len_range
    out = []
    for b in range(w.B):
        k = 0
        while True:
            L = uniform_int(w.seed, TID_LEN, b * 1000 + k, lo, hi)
            k += 1
            if L % MSA_BLOCK != 0:
                break
        out.append(L)
    return out


def needle_blocks_for(w: Workload, seq_lens: Sequence[int]) -> List[List[int]]:
    """Distinct needle block ids per sequence, uniform among full blocks that hold no query token."""
    out = []
    for b, L in enumerate(seq_lens):
        n_cand = (L - w.Tq) // MSA_BLOCK  # full blocks strictly before the first query token's block
        if w.needles == 0 or n_cand <= 0:
            out.append([])
            continue
        cand = torch.arange(n_cand, dtype=torch.int64).view(1, -1)
        h = hash_u32(w.seed, TID_NEEDLE, 3, torch.tensor([[b]]), cand).view(-1)
        order = torch.argsort(h * n_cand + cand.view(-1), stable=True)
        out.append(sorted(order[: min(w.needles, n_cand)].tolist()))
    return out


def tensor_scale_cal(amax: float) -> float:
    """Per-tensor NVFP4 scale from a calibrated amax: amax / (6 * 448), in float32."""
    import numpy as np
    return float(np.float32(amax) / np.float32(6.0 * 448.0))


@dataclass
class Inputs:
    """fp32 caches (before quantisation) + bf16 queries for one workload (or a slice of it)."""
    w: Workload
    seq_lens: List[int]
    needles: List[List[int]]
    q: torch.Tensor          # bf16 [B, Tq, Hq, D]
    q_idx: torch.Tensor      # bf16 [B, Tq, HI, DI]
    w_idx: Optional[torch.Tensor]  # fp32 [B, Tq, HI] or None
    k: Optional[torch.Tensor] = None   # fp32 [B, Hkv, lmax, D]
    v: Optional[torch.Tensor] = None   # fp32 [B, Hkv, lmax, D]
    ik: Optional[torch.Tensor] = None  # fp32 [B, 1, lmax, DI]
    s_k: float = 0.0
    s_v: float = 0.0
    s_ik: float = 0.0
    batch_ids: List[int] = field(default_factory=list)


def queries(w: Workload, batch_ids: Sequence[int], device="cpu"):
    """bf16 q [nb, Tq, Hq, D], q_idx [nb, Tq, HI, DI] and optional fp32 weights [nb, Tq, HI]."""
    qs, qis, ws = [], [], []
    for b in batch_ids:
        qs.append(normal_tensor(w.seed, TID_Q, w.Tq * w.Hq, w.D, device, row0=b * w.Tq * w.Hq)
                  .to(torch.bfloat16).view(w.Tq, w.Hq, w.D))
        qis.append(normal_tensor(w.seed, TID_QI, w.Tq * w.HI, w.DI, device, row0=b * w.Tq * w.HI)
                   .to(torch.bfloat16).view(w.Tq, w.HI, w.DI))
        if w.weights:
            ws.append(normal_tensor(w.seed, TID_W, w.Tq, w.HI, device, row0=b * w.Tq).abs())
    q = torch.stack(qs) if qs else torch.empty(0, w.Tq, w.Hq, w.D, dtype=torch.bfloat16, device=device)
    qi = torch.stack(qis) if qis else torch.empty(0, w.Tq, w.HI, w.DI, dtype=torch.bfloat16, device=device)
    wi = torch.stack(ws) if ws else None
    return q, qi, wi


def qbar(q_idx_b: torch.Tensor) -> torch.Tensor:
    """Mean over indexer heads of the committed (t = 0) token's query, fp32, fixed order."""
    HI = q_idx_b.shape[1]
    acc = q_idx_b[0, 0].to(torch.float32)
    for h in range(1, HI):
        acc = acc + q_idx_b[0, h].to(torch.float32)
    return acc * (1.0 / HI) if (HI & (HI - 1)) == 0 else acc / float(HI)


def cache_rows(w: Workload, b: int, h: int, heads: int) -> int:
    return (b * heads + h)


def kv_tokens(w: Workload, tid: int, b: int, heads: int, dim: int, t0: int, t1: int, device="cpu") -> torch.Tensor:
    """fp32 [heads, t1-t0, dim] of cache tensor ``tid`` (K or V) for sequence b, tokens [t0, t1)."""
    out = torch.empty(heads, t1 - t0, dim, dtype=torch.float32, device=device)
    for h in range(heads):
        # column index = token * dim + d keeps (row, col) unique per element
        flat = normal_tensor(w.seed, tid, 1, (t1 - t0) * dim, device, row0=b * heads + h, col0=t0 * dim)
        out[h] = flat.view(t1 - t0, dim)
    return out


def index_key_tokens(w: Workload, b: int, t0: int, t1: int, needles_b: Sequence[int],
                     qbar_b: Optional[torch.Tensor], device="cpu") -> torch.Tensor:
    """fp32 [1, t1-t0, DI] index keys of sequence b, tokens [t0, t1), needles applied."""
    ik = kv_tokens(w, TID_IK, b, 1, w.DI, t0, t1, device)
    if needles_b and qbar_b is not None:
        add = qbar_b.to(device) * 0.5
        for n in needles_b:
            a, c = max(t0, n * MSA_BLOCK), min(t1, (n + 1) * MSA_BLOCK)
            if a < c:
                ik[0, a - t0:c - t0] = ik[0, a - t0:c - t0] + add
    return ik


def make_inputs(w: Workload, batch_ids: Optional[Sequence[int]] = None, device="cpu",
                with_kv: bool = True) -> Inputs:
    """Full fp32 caches (length lmax, zero past L) + queries for the given sequences."""
    if batch_ids is None:
        batch_ids = list(range(w.B))
    lens_all = seq_lens_for(w)
    needles_all = needle_blocks_for(w, lens_all)
    q, qi, wi = queries(w, batch_ids, device)
    nb = len(batch_ids)
    ik = torch.zeros(nb, 1, w.lmax, w.DI, dtype=torch.float32, device=device)
    k = v = None
    if with_kv:
        k = torch.zeros(nb, w.Hkv, w.lmax, w.D, dtype=torch.float32, device=device)
        v = torch.zeros(nb, w.Hkv, w.lmax, w.D, dtype=torch.float32, device=device)
    for i, b in enumerate(batch_ids):
        L = lens_all[b]
        ik[i, :, :L] = index_key_tokens(w, b, 0, L, needles_all[b], qbar(qi[i]), device)
        if with_kv:
            k[i, :, :L] = kv_tokens(w, TID_K, b, w.Hkv, w.D, 0, L, device)
            v[i, :, :L] = kv_tokens(w, TID_V, b, w.Hkv, w.D, 0, L, device)
    s = tensor_scale_cal(w.amax_cal)
    return Inputs(w=w, seq_lens=[lens_all[b] for b in batch_ids], needles=[needles_all[b] for b in batch_ids],
                  q=q, q_idx=qi, w_idx=wi, k=k, v=v, ik=ik, s_k=s, s_v=s, s_ik=s, batch_ids=list(batch_ids))
