"""Seeded synthetic inputs for the fused QK-RMSNorm + RoPE path.

This module is shared by the tests, the bench and the oracle's callers. It
draws random tensors, builds position ids and packs documents into rows; it
holds none of the normalisation or rotary arithmetic, which lives separately
in the CUDA library and in the CPU oracle.

The five workloads are the shapes the pages care about:

* ``tiny`` -- a 32-token fp32 case small enough for exhaustive CPU checks.
* ``qwen2.5-0.5b`` -- Qwen2.5-0.5B attention shapes (14 query heads, 2 KV
  heads, head dim 64), the model Chronicals fine-tunes in its headline
  throughput figure (Chronicals, arXiv 2601.02609, abstract).
* ``llama3-8b-qknorm`` -- Llama-3-8B attention shapes with QK-norm added.
* ``partial-rope-64k`` -- a 65,536-token row with rotary on a quarter of each
  head ("Fractional Rotation, Full Potential? Investigating Performance and
  Convergence of Partial RoPE", abstract).
* ``bfd-packed`` -- documents of log-uniform length packed into 4096-token
  rows by Best-Fit Decreasing, position ids restarting at every document
  (Chronicals, abstract, contribution (4)).

Recipe (identical for every consumer): ``numpy.random.default_rng(seed)``
(PCG64) draws standard normals in float32 in the fixed order q, k, gamma_q,
gamma_k, dq_out, dk_out; q and k are multiplied by the workload's scale,
gamma is ``1 + 0.1 * N(0, 1)``; every tensor is then rounded once to the I/O
dtype with round-to-nearest-even. Both sides consume the rounded values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One problem instance: the shape, the rotary and norm constants, I/O dtype."""

    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    rotary_dim: int
    theta: float
    eps: float
    dtype: str  # "f32" or "bf16"
    qk_scale: float = 1.0
    # packed-sequence recipe (bfd-packed only)
    packed: bool = False
    total_tokens: int = 0
    row_cap: int = 0
    doc_len_range: tuple = (64, 4096)
    index: int = 0  # position in the workload list; seeds are 1000*index + k

    @property
    def T(self) -> int:
        return self.B * self.S

    @property
    def H(self) -> int:
        return self.Hq + self.Hkv

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny": Workload("tiny", B=1, S=32, Hq=4, Hkv=2, D=16, rotary_dim=16,
                     theta=1e4, eps=1e-6, dtype="f32", qk_scale=1.0, index=0),
    "qwen2.5-0.5b": Workload("qwen2.5-0.5b", B=8, S=2048, Hq=14, Hkv=2, D=64,
                             rotary_dim=64, theta=1e6, eps=1e-6, dtype="bf16",
                             qk_scale=3.0, index=1),
    "llama3-8b-qknorm": Workload("llama3-8b-qknorm", B=4, S=8192, Hq=32, Hkv=8,
                                 D=128, rotary_dim=128, theta=5e5, eps=1e-5,
                                 dtype="bf16", qk_scale=4.0, index=2),
    "partial-rope-64k": Workload("partial-rope-64k", B=1, S=65536, Hq=32, Hkv=8,
                                 D=128, rotary_dim=32, theta=1e6, eps=1e-6,
                                 dtype="bf16", qk_scale=1.0, index=3),
    # B is fixed by the packer (rows actually opened); S is the row capacity.
    "bfd-packed": Workload("bfd-packed", B=0, S=4096, Hq=16, Hkv=4, D=128,
                           rotary_dim=128, theta=1e4, eps=1e-6, dtype="bf16",
                           qk_scale=1.0, packed=True, total_tokens=16384,
                           row_cap=4096, doc_len_range=(64, 4096), index=4),
}

BENCH_WORKLOAD = "partial-rope-64k"


def seed_for(w: Workload, k: int = 0) -> int:
    return 1000 * w.index + k


# --------------------------------------------------------------------------
# Best-Fit-Decreasing packing (Chronicals, abstract, contribution (4)).
# --------------------------------------------------------------------------

def draw_doc_lengths(rng: np.random.Generator, total: int, lo: int, hi: int) -> list:
    """Log-uniform document lengths in [lo, hi], drawn until they sum to
    ``total``; the last one is cut to the remainder (it may fall below lo)."""
    lengths = []
    acc = 0
    while acc < total:
        L = int(round(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        L = max(1, min(L, total - acc))
        lengths.append(L)
        acc += L
    return lengths


def bfd_pack(lengths: list, cap: int) -> list:
    """Best-Fit Decreasing bin packing.

    Documents are taken longest first (ties keep draw order). Each goes into
    the open row whose remaining capacity is the smallest that still fits it
    (ties go to the lowest row index); when none fits, a new row is opened.
    Returns a list of rows, each a list of document indices in placement
    order.
    """
    if any(L > cap or L < 1 for L in lengths):
        raise ValueError("every document must have 1 <= length <= row capacity")
    order = sorted(range(len(lengths)), key=lambda i: (-lengths[i], i))
    rows: list = []
    free: list = []
    for i in order:
        L = lengths[i]
        best = -1
        for r, f in enumerate(free):
            if f >= L and (best < 0 or f < free[best]):
                best = r
        if best < 0:
            rows.append([i])
            free.append(cap - L)
        else:
            rows[best].append(i)
            free[best] -= L
    return rows


def packed_layout(lengths: list, rows: list, cap: int):
    """Slot layout of packed rows.

    Returns ``(pos, doc_id)``, both int32 arrays of shape [n_rows, cap]:
    ``pos`` restarts at 0 at every document and is 0 on padding slots;
    ``doc_id`` is the document index, or -1 on padding.
    """
    n = len(rows)
    pos = np.zeros((n, cap), dtype=np.int32)
    doc = np.full((n, cap), -1, dtype=np.int32)
    for r, docs in enumerate(rows):
        at = 0
        for i in docs:
            L = lengths[i]
            pos[r, at:at + L] = np.arange(L, dtype=np.int32)
            doc[r, at:at + L] = i
            at += L
    return pos, doc


# --------------------------------------------------------------------------
# Tensor generation
# --------------------------------------------------------------------------

@dataclass
class Inputs:
    """Host tensors of one problem, already rounded to the I/O dtype.

    Shapes: q [B,S,Hq,D], k [B,S,Hkv,D], gamma_q/gamma_k [D],
    dq_out/dk_out like q/k, pos [B,S] int32 or None (position = s).
    ``valid`` [B,S] bool marks real tokens (all True except packing pads).
    """

    w: Workload
    q: torch.Tensor
    k: torch.Tensor
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor
    dq_out: torch.Tensor
    dk_out: torch.Tensor
    pos: Optional[torch.Tensor]
    valid: torch.Tensor
    doc_lengths: list = field(default_factory=list)
    rows: list = field(default_factory=list)

    @property
    def real_tokens(self) -> int:
        return int(self.valid.sum())


def _normal(rng, shape, scale, torch_dtype, chunk=1 << 24):
    """float32 N(0,1)*scale drawn in C order, rounded once to torch_dtype."""
    out = torch.empty(shape, dtype=torch_dtype)
    flat = out.view(-1)
    n = flat.numel()
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        v = rng.standard_normal(b - a, dtype=np.float32)
        if scale != 1.0:
            v *= np.float32(scale)
        flat[a:b] = torch.from_numpy(v).to(torch_dtype)
    return out


def resolve(w: Workload, seed: int) -> tuple:
    """For packed workloads, the concrete (Workload with B set, lengths, rows)."""
    if not w.packed:
        return w, [], []
    drng = np.random.default_rng([seed, 1])
    lengths = draw_doc_lengths(drng, w.total_tokens, *w.doc_len_range)
    rows = bfd_pack(lengths, w.row_cap)
    return replace(w, B=len(rows), S=w.row_cap), lengths, rows


def make_inputs(w: Workload | str, seed: Optional[int] = None,
                with_grads: bool = True, **overrides) -> Inputs:
    """Seeded synthetic inputs for workload ``w`` (see the module recipe).

    ``overrides`` replace Workload fields (for small variants in tests).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if overrides:
        w = replace(w, **overrides)
    if seed is None:
        seed = seed_for(w)
    w, lengths, rows = resolve(w, seed)
    rng = np.random.default_rng(seed)
    td = w.torch_dtype
    q = _normal(rng, (w.B, w.S, w.Hq, w.D), w.qk_scale, td)
    k = _normal(rng, (w.B, w.S, w.Hkv, w.D), w.qk_scale, td)
    gq = (1.0 + 0.1 * rng.standard_normal(w.D)).astype(np.float32)
    gk = (1.0 + 0.1 * rng.standard_normal(w.D)).astype(np.float32)
    gamma_q = torch.from_numpy(gq).to(td)
    gamma_k = torch.from_numpy(gk).to(td)
    if with_grads:
        dq_out = _normal(rng, (w.B, w.S, w.Hq, w.D), 1.0, td)
        dk_out = _normal(rng, (w.B, w.S, w.Hkv, w.D), 1.0, td)
    else:
        dq_out = dk_out = None
    valid = torch.ones((w.B, w.S), dtype=torch.bool)
    pos = None
    if w.packed:
        p, doc = packed_layout(lengths, rows, w.S)
        pos = torch.from_numpy(p)
        valid = torch.from_numpy(doc >= 0)
        pad = ~valid
        # padding slots carry zeros in every per-token tensor
        q[pad] = 0
        k[pad] = 0
        if with_grads:
            dq_out[pad] = 0
            dk_out[pad] = 0
    return Inputs(w, q, k, gamma_q, gamma_k, dq_out, dk_out, pos, valid,
                  lengths, rows)


def layerwise_gamma(w: Workload, seed: int) -> tuple:
    """Full-hidden weights of the layerwise (all-heads) QK-norm: gamma_q
    [Hq*D], gamma_k [Hkv*D], each ``1 + 0.1 * N(0, 1)`` drawn in float32 from
    ``default_rng([seed, 2])`` (q first) and rounded once to the I/O dtype."""
    rng = np.random.default_rng([seed, 2])
    td = w.torch_dtype
    gq = (1.0 + 0.1 * rng.standard_normal(w.Hq * w.D)).astype(np.float32)
    gk = (1.0 + 0.1 * rng.standard_normal(w.Hkv * w.D)).astype(np.float32)
    return torch.from_numpy(gq).to(td), torch.from_numpy(gk).to(td)


def contract_bytes(w: Workload, with_pos: bool = False) -> dict:
    """Minimum HBM bytes each direction must move (per launch).

    fwd reads X and writes Y and the fp32 inverse RMS; bwd reads X, dY and
    the inverse RMS and writes dX. gamma / dgamma (a few hundred bytes) and,
    when given, the int32 position ids (4 B per token) are added too.
    """
    e = w.elem_bytes
    rows = w.T * w.H
    elems = rows * w.D
    g = 2 * w.D * e
    p = 4 * w.T if with_pos else 0
    fwd = 2 * elems * e + 4 * rows + g + p
    bwd = 3 * elems * e + 4 * rows + g + 2 * w.D * 4 + p
    return {"fwd": fwd, "bwd": bwd, "rows": rows, "elems": elems}
