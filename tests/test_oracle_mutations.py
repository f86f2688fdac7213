"""Plant plausible mistakes in a private copy of the oracle (CPU only) and
check that the pins catch each one.  Nothing here touches the real oracle."""
import importlib.util
import math
import os

import numpy as np
import pytest

from oracle_pins import ALL_CHECKS

ORACLE_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "gva_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("gva_oracle_mutant", ORACLE_FILE)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_rope_sign(m):
    orig = m.rope

    def bad(x, pos, base):                       # rotate the wrong way in one component
        y = orig(x, pos, base)
        half = np.asarray(x).shape[-1] // 2
        y[..., half:] = 2 * np.asarray(x, dtype=float)[..., half:] * np.cos(0) - y[..., half:]
        return y
    m.rope = bad


def _mut_rope_adjacent_pairs(m):
    def bad(x, pos, base):                       # interleaved pairs instead of rotate-half
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        if d == 0:
            return x.copy()
        inv = np.power(float(base), -np.arange(d // 2) * 2.0 / d)
        a = np.asarray(pos, dtype=np.float64)[..., None] * inv
        x1, x2 = x[..., 0::2], x[..., 1::2]
        y = np.empty_like(x)
        y[..., 0::2] = x1 * np.cos(a) - x2 * np.sin(a)
        y[..., 1::2] = x1 * np.sin(a) + x2 * np.cos(a)
        return y
    m.rope = bad


def _mut_rope_freq(m):
    orig = m.rope
    m.rope = lambda x, pos, base: orig(x, pos, base * 2.0)


def _mut_drop_rope_term(m):
    orig = m.gva_decode

    def bad(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, **kw):
        return orig(q, M, q_pos, V, np.zeros_like(np.asarray(k_rope, dtype=float)), seq_offset,
                    seq_len, d_n, d_r, base, **kw)
    m.gva_decode = bad


def _mut_group_map(m):
    orig = m.gva_decode

    def bad(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, **kw):
        V = np.asarray(V, dtype=float)
        G = V.shape[1]
        return orig(q, M, q_pos, V[:, ::-1, :] if G > 1 else V, k_rope, seq_offset, seq_len,
                    d_n, d_r, base, **kw)
    m.gva_decode = bad


def _mut_transposed_map(m):
    orig = m.gva_decode

    def bad(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, **kw):
        M = np.asarray(M, dtype=float)
        if M.shape[1] == M.shape[2]:
            M = M.transpose(0, 2, 1)
        else:   # cyclically shift the rows: a wrong index into M_h
            M = np.roll(M, 1, axis=1)
        return orig(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, **kw)
    m.gva_decode = bad


def _mut_scale(m):
    orig = m.gva_decode

    def bad(*a, **kw):
        kw["scale"] = 1.0 / math.sqrt(max(1, a[7] if len(a) > 7 else kw["d_n"]))
        return orig(*a, **kw)
    m.gva_decode = bad


def _mut_softmax_no_norm(m):
    orig = m._softmax_attend

    def bad(s, Vg):
        o, l = orig(s, Vg)
        return o * (1 + 1e-3 * len(s)), l
    m._softmax_attend = bad


def _mut_off_by_one_len(m):
    orig = m.gva_decode

    def bad(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, **kw):
        L = np.maximum(np.asarray(seq_len) - 1, 0)
        return orig(q, M, q_pos, V, k_rope, seq_offset, L, d_n, d_r, base, **kw)
    m.gva_decode = bad


def _mut_gqa_group_map(m):
    orig = m.gqa_decode

    def bad(q, K, V, seq_offset, seq_len, **kw):
        K = np.asarray(K, dtype=float)
        return orig(q, K[:, ::-1, :], V, seq_offset, seq_len, **kw)
    m.gqa_decode = bad


def _mut_bf16_truncate(m):
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        mm, e = np.frexp(x)
        return np.ldexp(np.trunc(mm * 256.0), e - 8)
    m.round_to_bf16 = bad


def _mut_cache_count(m):
    m.cache_scalars_gva = lambda T, G, d_h, d_r: T * G * d_h + T * G * d_r


def _mut_append_no_rotate(m):
    m_rope = m.rope
    orig = m.append_cache

    def bad(V, K, v, k, slot, pos, base, dtype):
        m.rope = lambda x, p, b: np.asarray(x, dtype=float)
        try:
            return orig(V, K, v, k, slot, pos, base, dtype)
        finally:
            m.rope = m_rope
    m.append_cache = bad


def _mut_gqa_append_no_rotate(m):
    orig = m.gqa_append_cache

    def bad(K_cache, V_cache, k_new, v_new, slot, pos, base, dtype):   # key stored unrotated
        return orig(K_cache, V_cache, k_new, v_new, slot, np.zeros_like(np.asarray(pos)), base, dtype)
    m.gqa_append_cache = bad


def _mut_causal_off_by_one(m):
    orig = m.gva_decode

    def multi(q, M, q_pos, V, k_rope, seq_offset, seq_len, d_n, d_r, base, scale=None):
        q = np.asarray(q, dtype=float)
        Q = q.shape[1]
        outs, lses = [], []
        for i in range(Q):                       # sees one row past its own position
            Li = np.minimum(np.asarray(seq_len) - Q + i + 2, np.asarray(seq_len))
            o, l = orig(q[:, i], M, np.asarray(q_pos)[:, i], V, k_rope, seq_offset, Li, d_n, d_r,
                        base, scale=scale)
            outs.append(o)
            lses.append(l)
        return np.stack(outs, 1), np.stack(lses, 1)
    m.gva_decode_multi = multi


MUTATIONS = [_mut_rope_sign, _mut_rope_adjacent_pairs, _mut_rope_freq, _mut_drop_rope_term,
             _mut_group_map, _mut_transposed_map, _mut_scale, _mut_softmax_no_norm,
             _mut_off_by_one_len, _mut_gqa_group_map, _mut_bf16_truncate, _mut_cache_count,
             _mut_append_no_rotate, _mut_causal_off_by_one, _mut_gqa_append_no_rotate]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__[5:])
def test_pins_catch_planted_mistake(mutate):
    m = fresh_oracle()
    mutate(m)
    failed = []
    for check in ALL_CHECKS:
        try:
            check(m)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught {mutate.__name__}"
