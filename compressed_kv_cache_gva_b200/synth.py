"""Seeded synthetic workloads for GVA decode.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no RoPE, no absorption, no softmax). Both the CUDA path and
the float64 oracle are fed from the arrays it returns, so the two sides always
see bit-identical inputs.

Recipe (one ``numpy.random.default_rng(seed)`` stream, draws in this fixed
order): cache lengths (ragged workloads only, uniform integers, both ends
inclusive), then q, M, V, k_rope, each drawn as float32 standard normals;
M is scaled by 1/sqrt(d_h) so that M_h ~ N(0, 1/d_h) elementwise.  For bf16
workloads every tensor is rounded to bf16 (round-to-nearest-even) on the host
once, and both sides receive the rounded values.

The k_rope array stands for the cached positional key.  Rotation by RoPE is
orthogonal, so an i.i.d. N(0,1) vector stays i.i.d. N(0,1) after rotation: the
same draw serves as the raw (unrotated) key for append tests and as the stored
(rotated) cache for decode tests.

Cache layout: slots [S, G, d_h] for V and [S, d_r] for k_rope; sequence b owns
slots seq_offset[b] .. seq_offset[b] + capacity_b - 1, packed back to back,
where capacity_b = seq_len[b] + extra_slots (room for appended tokens).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one GVA decode step (one query token per sequence)."""

    name: str
    B: int
    H: int
    G: int
    d_h: int
    d_n: int
    d_r: int
    T: int                      # cache length per sequence (fixed-length workloads)
    rope_base: float
    dtype: str                  # "f32" or "bf16": cache, query and M storage type
    ragged: Optional[tuple] = None   # (lo, hi) inclusive bounds for U{lo..hi} lengths
    seed: int = 0

    @property
    def hpg(self) -> int:
        return self.H // self.G

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the GVA decode study (shapes, distributions and seeds).
WORKLOADS = {
    # tiny correctness case, fp32
    "tiny_fp32_t64": Workload("tiny_fp32_t64", B=1, H=4, G=2, d_h=32, d_n=24, d_r=8,
                              T=64, rope_base=10000.0, dtype="f32"),
    # 350M-class head shape
    "350m_b8_t4096": Workload("350m_b8_t4096", B=8, H=16, G=4, d_h=64, d_n=48, d_r=16,
                              T=4096, rope_base=10000.0, dtype="bf16"),
    # wider positional slice, long context (also run as same-shape GQA)
    "dr24_b4_t32768": Workload("dr24_b4_t32768", B=4, H=16, G=4, d_h=64, d_n=40, d_r=24,
                               T=32768, rope_base=10000.0, dtype="bf16"),
    # ragged serving batch: 64 sequences with lengths U{1024..16384}
    "ragged_b64_1k_16k": Workload("ragged_b64_1k_16k", B=64, H=16, G=4, d_h=64, d_n=48,
                                  d_r=16, T=16384, rope_base=10000.0, dtype="bf16",
                                  ragged=(1024, 16384)),
    # large-model head shape, very long context
    "d128_b1_t131072": Workload("d128_b1_t131072", B=1, H=32, G=8, d_h=128, d_n=112,
                                d_r=16, T=131072, rope_base=500000.0, dtype="bf16"),
}


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t if dtype == "f32" else t.to(torch.bfloat16)


@dataclasses.dataclass
class DecodeInputs:
    """Host tensors of one decode step (CPU, storage dtype of the workload)."""

    wl: Workload
    seq_len: torch.Tensor      # int32 [B]
    seq_offset: torch.Tensor   # int32 [B]
    q_pos: torch.Tensor        # int32 [B] position of the query token
    q: torch.Tensor            # [B, H, d_n + d_r]  (content slice first, rope slice last)
    M: torch.Tensor            # [H, d_h, d_n]
    V: torch.Tensor            # [S, G, d_h]
    k_rope: torch.Tensor       # [S, d_r]  (stored, i.e. already rotated)
    num_slots: int

    @property
    def total_tokens(self) -> int:
        return int(self.seq_len.to(torch.int64).sum())


def lengths_for(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    if wl.ragged is None:
        return np.full(wl.B, wl.T, dtype=np.int64)
    lo, hi = wl.ragged
    return rng.integers(lo, hi, size=wl.B, endpoint=True).astype(np.int64)


def make_decode_inputs(wl: Workload, extra_slots: int = 0,
                       lengths: Optional[np.ndarray] = None) -> DecodeInputs:
    """Draw one decode step's inputs.  ``lengths`` overrides the drawn lengths
    (edge-case tests); the query position defaults to the cache length."""
    rng = np.random.default_rng(wl.seed)
    drawn = lengths_for(wl, rng)
    L = drawn if lengths is None else np.asarray(lengths, dtype=np.int64)
    B = len(L)
    cap = L + extra_slots
    offs = np.concatenate([[0], np.cumsum(cap)[:-1]]).astype(np.int64)
    S = int(cap.sum())
    f32 = np.float32
    q = rng.standard_normal((B, wl.H, wl.d_n + wl.d_r), dtype=f32)
    M = rng.standard_normal((wl.H, wl.d_h, wl.d_n), dtype=f32) * f32(1.0 / np.sqrt(wl.d_h))
    V = rng.standard_normal((max(S, 1), wl.G, wl.d_h), dtype=f32)
    kr = rng.standard_normal((max(S, 1), wl.d_r), dtype=f32)
    return DecodeInputs(
        wl=wl,
        seq_len=torch.from_numpy(L.astype(np.int32)),
        seq_offset=torch.from_numpy(offs.astype(np.int32)),
        q_pos=torch.from_numpy(L.astype(np.int32)),
        q=_round(q, wl.dtype), M=_round(M, wl.dtype),
        V=_round(V, wl.dtype), k_rope=_round(kr, wl.dtype),
        num_slots=max(S, 1),
    )


@dataclasses.dataclass
class AppendInputs:
    v_new: torch.Tensor     # [N, G, d_h]
    kpe_new: torch.Tensor   # [N, d_r] raw (unrotated) positional key
    slot: torch.Tensor      # int32 [N]
    pos: torch.Tensor       # int32 [N]


def make_append_inputs(wl: Workload, slot: np.ndarray, pos: np.ndarray,
                       seed: int = 1) -> AppendInputs:
    rng = np.random.default_rng(seed)
    N = len(slot)
    f32 = np.float32
    v = rng.standard_normal((N, wl.G, wl.d_h), dtype=f32)
    k = rng.standard_normal((N, wl.d_r), dtype=f32)
    return AppendInputs(v_new=_round(v, wl.dtype), kpe_new=_round(k, wl.dtype),
                        slot=torch.from_numpy(np.asarray(slot, dtype=np.int32)),
                        pos=torch.from_numpy(np.asarray(pos, dtype=np.int32)))


@dataclasses.dataclass
class GQAInputs:
    """Same-shape GQA cache: K and V both [S, G, d_h]; q [B, H, d_h] (keys and
    query already rotated, so they are plain N(0,1) draws)."""

    seq_len: torch.Tensor
    seq_offset: torch.Tensor
    q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    num_slots: int


def make_gqa_inputs(wl: Workload, extra_slots: int = 0,
                    lengths: Optional[np.ndarray] = None) -> GQAInputs:
    rng = np.random.default_rng(wl.seed + 1000)
    drawn = lengths_for(wl, rng)
    L = drawn if lengths is None else np.asarray(lengths, dtype=np.int64)
    cap = L + extra_slots
    offs = np.concatenate([[0], np.cumsum(cap)[:-1]]).astype(np.int64)
    S = max(int(cap.sum()), 1)
    f32 = np.float32
    q = rng.standard_normal((len(L), wl.H, wl.d_h), dtype=f32)
    K = rng.standard_normal((S, wl.G, wl.d_h), dtype=f32)
    V = rng.standard_normal((S, wl.G, wl.d_h), dtype=f32)
    return GQAInputs(seq_len=torch.from_numpy(L.astype(np.int32)),
                     seq_offset=torch.from_numpy(offs.astype(np.int32)),
                     q=_round(q, wl.dtype), K=_round(K, wl.dtype), V=_round(V, wl.dtype),
                     num_slots=S)


@dataclasses.dataclass
class GQAAppendInputs:
    k_new: torch.Tensor     # [N, G, d_h] raw (unrotated) key
    v_new: torch.Tensor     # [N, G, d_h]
    slot: torch.Tensor      # int32 [N]
    pos: torch.Tensor       # int32 [N]


def make_gqa_append_inputs(wl: Workload, slot: np.ndarray, pos: np.ndarray,
                           seed: int = 3) -> GQAAppendInputs:
    """New tokens for the same-shape GQA cache: key and value rows drawn as float32
    standard normals (key first), rounded to the workload's storage type."""
    rng = np.random.default_rng(seed)
    N = len(slot)
    f32 = np.float32
    k = rng.standard_normal((N, wl.G, wl.d_h), dtype=f32)
    v = rng.standard_normal((N, wl.G, wl.d_h), dtype=f32)
    return GQAAppendInputs(k_new=_round(k, wl.dtype), v_new=_round(v, wl.dtype),
                           slot=torch.from_numpy(np.asarray(slot, dtype=np.int32)),
                           pos=torch.from_numpy(np.asarray(pos, dtype=np.int32)))


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a stored tensor to float64 for the oracle."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def make_multi_queries(wl: Workload, B: int, n_query: int, seed: int = 2) -> torch.Tensor:
    """Queries of n_query new tokens per sequence, [B, n_query, H, d_n + d_r],
    float32 standard normals rounded to the workload's storage type."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, n_query, wl.H, wl.d_n + wl.d_r), dtype=np.float32)
    return _round(q, wl.dtype)
