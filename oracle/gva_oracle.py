"""Float64 CPU oracle for Grouped Value Attention (GVA) decode.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The CUDA library never calls it and
shares no code with it; the two meet only through the seeded inputs.

What it computes follows the pages on GVA ("Grouped Value Attention: Efficient
KV Caching via On-Demand Key Reconstruction", Tripathi, Kumar, Khan; the onedev.kr
review "GVA는 값만 캐시하고 키를 필요할 때 복원해 GQA 캐시를 절반으로 줄인다", the
bisque.today explainer "Grouped Value Attention matches GQA on a 47% smaller KV
cache", and the agihunt.info summary).  It deliberately takes the NON-absorbed
route: the content key K_h = V_g(h) M_h is materialised for every cached token,
the positional query is rotated, and plain softmax attention runs on the sum of
the two score terms.  The GPU path instead folds M_h into the query; the review's
"How it works" section (어떻게 동작하나) states that the two routes give the same
score exactly, so agreement between them is the parity claim.

Readings where the pages are silent:
  * softmax scale 1/sqrt(d_n + d_r);
  * RoPE pairs dimension i with i + d_r/2 ("rotate half"), frequency
    theta_i = base^(-2i/d_r), angle = position * theta_i evaluated in float64;
  * head-to-group map g(h) = h // (H/G);
  * the query vector is [content slice (d_n) | positional slice (d_r)];
  * the cache rows of sequence b sit at positions 0..L_b-1 and are all attended;
    the query's own position is an explicit input;
  * an empty sequence (L_b = 0) gives a zero output and lse = -inf;
  * the stored positional key is the exact rotation rounded once to the cache
    type (round to nearest, ties to even);
  * the matched GQA baseline rotates its whole key (and query) of width d_h the
    same way, pair i with i + d_h/2.

Every function is plain numpy in float64: per (sequence, head) loops around
library matmuls, no blocking, no fusion, no reordering beyond the definitions.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# Cache size counts
# ----------------------------------------------------------------------------

def cache_scalars_gva(T: int, G: int, d_h: int, d_r: int) -> int:
    """Persistent cache scalars of GVA with a decoupled shared positional key:
    N_GVA = T*G*d_h + T*d_r (onedev.kr review, section "What differs"
    (무엇과 다른가): grouped values plus one shared k_rope of width d_r)."""
    return T * G * d_h + T * d_r


def cache_scalars_gqa(T: int, G: int, d_h: int) -> int:
    """Matched GQA stores a key and a value per group: N_GQA = 2*T*G*d_h
    (same section of the onedev.kr review)."""
    return 2 * T * G * d_h


# ----------------------------------------------------------------------------
# Rounding to the cache storage type
# ----------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values once to the nearest bfloat16 value, ties to even,
    and return them as float64.  bfloat16 keeps 8 significant bits (1 implicit
    + 7 stored) and float32's exponent range (normal numbers from 2^-126,
    subnormal spacing 2^-133)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    m, e = np.frexp(x[nz])             # x = m * 2^e with 0.5 <= |m| < 1
    # spacing of bf16 values around x: 2^(e-8) for normals, 2^-133 below 2^-126
    q_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(x[nz], -q_exp)   # exact: only the exponent changes
    out[nz] = np.ldexp(np.rint(scaled), q_exp)   # np.rint rounds half to even
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    big = np.abs(out) > 3.3895313892515355e38    # largest finite bfloat16
    out[big] = np.sign(out[big]) * np.inf
    return out


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# RoPE on the decoupled positional slice
# ----------------------------------------------------------------------------

def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate the last axis of ``x`` (width d_r, even) by position ``pos``.

    The pages fix only that the positional key is k_rope = (x_j W_r) R_j^T with a
    position-dependent rotation R_j, and that R_t^T R_j = R_(j-t) (onedev.kr review,
    "What differs").  The concrete R is our reading: pair i with i + d_r/2 and
    rotate that pair by angle pos * base^(-2i/d_r)."""
    x = np.asarray(x, dtype=np.float64)
    d_r = x.shape[-1]
    if d_r == 0:
        return x.copy()
    assert d_r % 2 == 0
    half = d_r // 2
    inv_freq = np.power(float(base), -np.arange(half, dtype=np.float64) * 2.0 / d_r)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


# ----------------------------------------------------------------------------
# Absorbed query (the quantity the pages say is computed once per token per head)
# ----------------------------------------------------------------------------

def absorbed_query(q: np.ndarray, M: np.ndarray, q_pos: np.ndarray, d_n: int, d_r: int,
                   base: float) -> Tuple[np.ndarray, np.ndarray]:
    """q~_h = q_h^nope M_h^T and the rotated positional query.

    onedev.kr review, "How it works": q_h k_{j,h}^T = q_h (v_j M_h)^T
    = (q_h M_h^T) v_j^T = q~_h v_j^T with q~_h = q_h M_h^T computed once per query
    token and head.  Returns (q~ [B,H,d_h], RoPE(q_rope, q_pos) [B,H,d_r]),
    both unscaled, float64."""
    q = np.asarray(q, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    B, H, _ = q.shape
    d_h = M.shape[1]
    qt = np.empty((B, H, d_h))
    for h in range(H):
        qt[:, h, :] = q[:, h, :d_n] @ M[h].T
    qr = rope(q[:, :, d_n:d_n + d_r], np.asarray(q_pos)[:, None], base)
    return qt, qr


# ----------------------------------------------------------------------------
# Cache append
# ----------------------------------------------------------------------------

def append_cache(V_cache: np.ndarray, kr_cache: np.ndarray, v_new: np.ndarray,
                 kpe_new: np.ndarray, slot: np.ndarray, pos: np.ndarray, base: float,
                 dtype: str) -> Tuple[np.ndarray, np.ndarray, int]:
    """Write new tokens into the persistent cache: the grouped value unchanged,
    the positional key rotated by its own position and stored in the cache type
    (onedev.kr review, "What differs": k_rope = (x_j W_r) R_j^T, cached separately
    and shared by all heads).  Slots outside [0, S) are skipped and reported
    through the returned error flag.  Returns new copies of both caches."""
    V = np.array(V_cache, dtype=np.float64, copy=True)
    KR = np.array(kr_cache, dtype=np.float64, copy=True)
    S = V.shape[0]
    err = 0
    for i in range(len(slot)):
        s = int(slot[i])
        if s < 0 or s >= S:
            err = 1
            continue
        V[s] = np.asarray(v_new[i], dtype=np.float64)
        KR[s] = round_to_storage(rope(np.asarray(kpe_new[i], dtype=np.float64),
                                      float(pos[i]), base), dtype)
    return V, KR, err


def gqa_append_cache(K_cache: np.ndarray, V_cache: np.ndarray, k_new: np.ndarray,
                     v_new: np.ndarray, slot: np.ndarray, pos: np.ndarray, base: float,
                     dtype: str) -> Tuple[np.ndarray, np.ndarray, int]:
    """Append for the matched GQA baseline, which caches a key and a value per
    group and token (onedev.kr review, "What differs": N_GQA = 2*T*G*d_h).  Plain
    RoPE acts on the whole key, so every group's key of width d_h is rotated by
    the token's position (the same rotation as ``rope``, over d_h) and stored in
    the cache type; the value is stored unchanged.  Slots outside [0, S) are
    skipped and reported through the returned flag.  Returns new copies of K and V."""
    K = np.array(K_cache, dtype=np.float64, copy=True)
    V = np.array(V_cache, dtype=np.float64, copy=True)
    S = K.shape[0]
    err = 0
    for i in range(len(slot)):
        s = int(slot[i])
        if s < 0 or s >= S:
            err = 1
            continue
        V[s] = np.asarray(v_new[i], dtype=np.float64)
        K[s] = round_to_storage(rope(np.asarray(k_new[i], dtype=np.float64), float(pos[i]), base),
                                dtype)
    return K, V, err


# ----------------------------------------------------------------------------
# Decode attention, non-absorbed route
# ----------------------------------------------------------------------------

def _softmax_attend(s: np.ndarray, Vg: np.ndarray) -> Tuple[np.ndarray, float]:
    """softmax over the cache axis and the weighted sum of value rows; returns
    (output, natural-log log-sum-exp of the scores)."""
    if s.shape[0] == 0:
        return np.zeros(Vg.shape[1]), -math.inf
    mx = s.max()
    e = np.exp(s - mx)
    z = e.sum()
    return (e / z) @ Vg, float(mx + math.log(z))


def gva_decode(q: np.ndarray, M: np.ndarray, q_pos: np.ndarray, V: np.ndarray,
               k_rope: np.ndarray, seq_offset: np.ndarray, seq_len: np.ndarray,
               d_n: int, d_r: int, base: float, scale: Optional[float] = None,
               pairs: Optional[Iterable[Tuple[int, int]]] = None,
               return_probs: bool = False):
    """One GVA decode step by the non-absorbed route.

    For each sequence b and query head h (group g = h // (H/G)):
      K_n[j] = V[b, j, g, :] @ M_h              content key, materialised
                                                (onedev.kr review, "How it works": K_h = V_g(h) M_h)
      q_r'   = RoPE(q_rope, q_pos[b])            the stored k_rope is already rotated
      s_j    = (q_nope . K_n[j] + q_r' . k_rope[j]) * scale,  scale = 1/sqrt(d_n + d_r)
      o      = softmax(s) @ V[b, :, g, :]        values deliver the output
                                                (agihunt summary; onedev.kr review)
    Inputs are the stored values (already rounded to the cache type) as float64.
    ``pairs`` restricts the work to a list of (b, h); other outputs are NaN.
    Returns (out [B,H,d_h], lse [B,H]) and, with ``return_probs``, a dict of the
    softmax rows keyed by (b, h)."""
    q = np.asarray(q, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    KR = np.asarray(k_rope, dtype=np.float64)
    B, H, _ = q.shape
    G, d_h = V.shape[1], V.shape[2]
    hpg = H // G
    if scale is None:
        scale = 1.0 / math.sqrt(d_n + d_r)
    out = np.full((B, H, d_h), np.nan)
    lse = np.full((B, H), np.nan)
    probs = {}
    todo = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
    for b, h in todo:
        g = h // hpg
        L = int(seq_len[b])
        o0 = int(seq_offset[b])
        Vg = V[o0:o0 + L, g, :]                          # [L, d_h]
        Kn = Vg @ M[h]                                   # [L, d_n]
        qn = q[b, h, :d_n]
        qr = rope(q[b, h, d_n:d_n + d_r], float(q_pos[b]), base)
        s = (Kn @ qn + KR[o0:o0 + L, :d_r] @ qr) * scale
        out[b, h], lse[b, h] = _softmax_attend(s, Vg)
        if return_probs:
            probs[(b, h)] = np.exp(s - lse[b, h]) if L else s
    if return_probs:
        return out, lse, probs
    return out, lse


def gqa_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray, seq_offset: np.ndarray,
               seq_len: np.ndarray, scale: Optional[float] = None,
               pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Same-shape grouped-query attention decode (the matched baseline in every
    page): each group caches a key and a value per token, heads of a group share
    them, s_j = q_h . K[j, g] * scale with scale = 1/sqrt(d_h), keys and query
    given already rotated."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, d_h = q.shape
    G = K.shape[1]
    hpg = H // G
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    out = np.full((B, H, d_h), np.nan)
    lse = np.full((B, H), np.nan)
    todo = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
    for b, h in todo:
        g = h // hpg
        L = int(seq_len[b])
        o0 = int(seq_offset[b])
        s = (K[o0:o0 + L, g, :] @ q[b, h]) * scale
        out[b, h], lse[b, h] = _softmax_attend(s, V[o0:o0 + L, g, :])
    return out, lse


def gva_decode_multi(q: np.ndarray, M: np.ndarray, q_pos: np.ndarray, V: np.ndarray,
                     k_rope: np.ndarray, seq_offset: np.ndarray, seq_len: np.ndarray, d_n: int,
                     d_r: int, base: float, scale: Optional[float] = None):
    """Decode of Q new tokens per sequence at once, causal among them.

    q [B, Q, H, d_n + d_r], q_pos [B, Q].  The Q new tokens are the last Q cache
    rows of each sequence (positions L-Q .. L-1, L = seq_len[b]); query i attends
    rows 0 .. L-Q+i, i.e. exactly what a one-token decode at that point of the
    sequence would see.  Returns (out [B,Q,H,d_h], lse [B,Q,H])."""
    q = np.asarray(q, dtype=np.float64)
    B, Q = q.shape[0], q.shape[1]
    L = np.asarray(seq_len, dtype=np.int64)
    outs, lses = [], []
    for i in range(Q):
        Li = np.maximum(L - Q + i + 1, 0)
        o, l = gva_decode(q[:, i], M, np.asarray(q_pos)[:, i], V, k_rope, seq_offset, Li, d_n, d_r,
                          base, scale=scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs, axis=1), np.stack(lses, axis=1)
