"""Pins of the float64 oracle to facts outside itself.

Each ``check_*`` takes an oracle module and raises AssertionError on a
mismatch.  ``test_oracle_pins.py`` runs them on the real oracle; the mutation
test runs them on copies with a planted mistake and expects at least one to fail.

What each pin rests on:
  * cache counts and ratio: the numbers the pages print (tests/golden/cache_ratio.txt);
  * K = V special case: torch's scaled_dot_product_attention (a library routine);
  * GQA oracle: the same library routine with grouped heads;
  * RoPE convention: transformers' Llama rotary embedding (library routine);
  * relative position: R_t^T R_j = R_(j-t) (onedev.kr review, "What differs");
  * absorption: the identity q (v M)^T = (q M^T) v^T, exact by the pages;
  * softmax closed forms: L = 1 returns the row, q = 0 returns the mean;
  * brute force: scalar loops on T <= 8.
"""
import math
import os

import numpy as np
import torch

from bruteforce import gva_decode_loops

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_case(rng, B=2, H=4, G=2, d_h=8, d_n=6, d_r=4, lens=(5, 3), extra=1):
    lens = np.asarray(lens)
    cap = lens + extra
    offs = np.concatenate([[0], np.cumsum(cap)[:-1]])
    S = int(cap.sum())
    q = rng.standard_normal((B, H, d_n + d_r))
    M = rng.standard_normal((H, d_h, d_n)) / math.sqrt(d_h)
    V = rng.standard_normal((S, G, d_h))
    KR = rng.standard_normal((S, d_r))
    return dict(q=q, M=M, q_pos=lens.copy(), V=V, k_rope=KR, seq_offset=offs, seq_len=lens,
                d_n=d_n, d_r=d_r)


# ---------------------------------------------------------------- page numbers

def check_cache_ratio(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "cache_ratio.txt"))
            if l.strip() and not l.startswith("#")]
    for gdh, d_r, saving, kind in rows:
        gdh, d_r, saving = int(gdh), int(d_r), float(saving)
        G, d_h, T = 4, gdh // 4, 4096
        n_gva = orc.cache_scalars_gva(T, G, d_h, d_r)
        n_gqa = orc.cache_scalars_gqa(T, G, d_h)
        ratio = n_gva / n_gqa
        # the closed form printed by the onedev.kr review
        assert abs(ratio - (0.5 + d_r / (2 * G * d_h))) < 1e-15, (gdh, d_r, ratio)
        if kind == "exact":
            assert abs((1 - ratio) - saving) < 1e-15
        else:
            assert abs((1 - ratio) - saving) < 0.01, (gdh, d_r, 1 - ratio, saving)


# ---------------------------------------------------------------- library routines

def _sdpa(q, k, v, scale):
    """q [B,H,1,d], k/v [B,H,L,d] float64 via torch's reference attention."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=scale).numpy()


def check_kv_shared_is_sdpa(orc):
    """M_h = I and d_r = 0: the content key is the value itself (the Shared-KV
    first attempt), i.e. textbook attention with K = V."""
    rng = np.random.default_rng(11)
    B, H, G, d_h, L = 1, 6, 3, 8, 7
    c = _rand_case(rng, B=B, H=H, G=G, d_h=d_h, d_n=d_h, d_r=0, lens=(L,), extra=0)
    c["M"] = np.broadcast_to(np.eye(d_h), (H, d_h, d_h)).copy()
    out, lse = orc.gva_decode(base=10000.0, **c)
    Vg = c["V"][:L]                                     # [L, G, d]
    # contiguous grouping: head h reads value group h // (H/G)
    kv = np.stack([Vg[:, h // (H // G), :] for h in range(H)])[None]   # [1,H,L,d]
    ref = _sdpa(c["q"][:, :, None, :], kv, kv, 1.0 / math.sqrt(d_h))[:, :, 0, :]
    assert np.max(np.abs(out - ref)) < 1e-12, np.max(np.abs(out - ref))


def check_gqa_is_sdpa(orc):
    rng = np.random.default_rng(12)
    B, H, G, d, lens = 2, 8, 2, 16, (9, 4)
    offs = np.array([0, 12])
    S = 20
    q = rng.standard_normal((B, H, d))
    K = rng.standard_normal((S, G, d))
    V = rng.standard_normal((S, G, d))
    out, lse = orc.gqa_decode(q, K, V, offs, np.array(lens))
    for b in range(B):
        L = lens[b]
        k = np.stack([K[offs[b]:offs[b] + L, h // (H // G)] for h in range(H)])[None]
        v = np.stack([V[offs[b]:offs[b] + L, h // (H // G)] for h in range(H)])[None]
        ref = _sdpa(q[b][None, :, None, :], k, v, 1.0 / math.sqrt(d))[0, :, 0, :]
        assert np.max(np.abs(out[b] - ref)) < 1e-12
        s = np.einsum("hd,hld->hl", q[b], k[0]) / math.sqrt(d)
        ref_lse = np.log(np.exp(s).sum(-1))
        assert np.max(np.abs(lse[b] - ref_lse)) < 1e-12


def check_rope_matches_llama(orc):
    """The rotate-half pairing and theta_i = base^(-2i/d_r) of the common Llama
    rotary embedding (transformers computes its angles in float32, hence the
    tolerance)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    rng = np.random.default_rng(13)
    for d_r, base in ((8, 10000.0), (16, 10000.0), (24, 10000.0), (16, 500000.0)):
        cfg = LlamaConfig(hidden_size=4 * d_r, num_attention_heads=4, head_dim=d_r, rope_theta=base)
        emb = LlamaRotaryEmbedding(cfg)
        pos = np.array([0, 1, 2, 7, 33, 64])
        x = rng.standard_normal((len(pos), d_r))
        xt = torch.from_numpy(x)[None, None]                       # [1,1,P,d]
        cos, sin = emb(xt, torch.from_numpy(pos)[None])
        ref, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
        got = orc.rope(x, pos, base)
        assert np.max(np.abs(got - ref[0, 0].numpy())) < 2e-5, (d_r, base)


# ---------------------------------------------------------------- invariants

def check_relative_position(orc):
    """Shifting every position (query and all keys) by the same amount leaves
    the output unchanged, because the score only sees R_t^T R_j = R_(j-t)."""
    rng = np.random.default_rng(14)
    c = _rand_case(rng, B=1, H=4, G=2, d_h=8, d_n=6, d_r=6, lens=(6,), extra=0)
    raw = c["k_rope"].copy()
    outs = []
    for shift in (0, 5, 1000):
        pos = np.arange(6) + shift
        c["k_rope"] = orc.rope(raw, pos, 10000.0)
        c["q_pos"] = np.array([6 + shift])
        outs.append(orc.gva_decode(base=10000.0, **c)[0])
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) < 1e-10
    # and the rotation is not trivial: a shift of the query alone changes it
    c["q_pos"] = np.array([3])
    moved = orc.gva_decode(base=10000.0, **c)[0]
    assert np.max(np.abs(moved - outs[-1])) > 1e-3


def check_rope_group_law(orc):
    """Rotation by p then by -p is the identity; position 0 is the identity;
    rotations compose additively and preserve the norm."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal((5, 16))
    for base in (10000.0, 500000.0):
        assert np.allclose(orc.rope(x, 0.0, base), x, atol=0, rtol=0)
        p = np.array([1.0, 17.0, 4095.0, 65536.0, 131072.0])
        y = orc.rope(x, p, base)
        assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
        assert np.max(np.abs(orc.rope(y, -p, base) - x)) < 1e-9
        assert np.max(np.abs(orc.rope(orc.rope(x, 3.0, base), 4.0, base) - orc.rope(x, 7.0, base))) < 1e-12
    # first pair (theta_0 = 1) of a unit vector at position p lands at angle p
    e0 = np.zeros(16)
    e0[0] = 1.0
    y = orc.rope(e0, 2.0, 10000.0)
    assert abs(y[0] - math.cos(2.0)) < 1e-15 and abs(y[8] - math.sin(2.0)) < 1e-15


def check_absorption_identity(orc):
    """Scores through the materialised key V M_h equal scores through the absorbed
    query q M_h^T, for every head, on random inputs (exact up to rounding)."""
    rng = np.random.default_rng(16)
    c = _rand_case(rng, B=2, H=6, G=3, d_h=10, d_n=7, d_r=4, lens=(6, 4), extra=2)
    out, lse = orc.gva_decode(base=10000.0, **c)
    qt, qr = orc.absorbed_query(c["q"], c["M"], c["q_pos"], c["d_n"], c["d_r"], 10000.0)
    scale = 1.0 / math.sqrt(c["d_n"] + c["d_r"])
    for b in range(2):
        L, o0 = c["seq_len"][b], c["seq_offset"][b]
        for h in range(6):
            g = h // 2
            Vg = c["V"][o0:o0 + L, g]
            s = (Vg @ qt[b, h] + c["k_rope"][o0:o0 + L] @ qr[b, h]) * scale
            p = np.exp(s - s.max())
            ref = (p / p.sum()) @ Vg
            assert np.max(np.abs(out[b, h] - ref)) < 1e-12
            assert abs(lse[b, h] - (s.max() + math.log(p.sum()))) < 1e-12


def check_softmax_closed_forms(orc):
    rng = np.random.default_rng(17)
    c = _rand_case(rng, B=3, H=4, G=2, d_h=8, d_n=5, d_r=4, lens=(1, 9, 0), extra=0)
    out, lse, probs = orc.gva_decode(base=10000.0, return_probs=True, **c)
    # L = 1: the single value row, exactly, and lse = the single score
    for h in range(4):
        assert np.array_equal(out[0, h], c["V"][0, h // 2])
    # L = 0: zero output, lse = -inf
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))
    # rows of softmax sum to one; output is a convex combination of value rows
    for (b, h), p in probs.items():
        if c["seq_len"][b] == 0:
            continue
        assert abs(p.sum() - 1) < 1e-13 and np.all(p >= 0)
        o0, L = c["seq_offset"][b], c["seq_len"][b]
        Vg = c["V"][o0:o0 + L, h // 2]
        assert np.all(out[b, h] <= Vg.max(0) + 1e-12) and np.all(out[b, h] >= Vg.min(0) - 1e-12)
    # q = 0: uniform attention, the output is the mean of the value rows
    c["q"] = np.zeros_like(c["q"])
    out0, lse0 = orc.gva_decode(base=10000.0, **c)
    Vg = c["V"][1:10]
    for h in range(4):
        assert np.max(np.abs(out0[1, h] - Vg[:, h // 2].mean(0))) < 1e-14
        assert abs(lse0[1, h] - math.log(9)) < 1e-14


def check_bruteforce(orc):
    """Scalar loops (no BLAS) agree with the oracle to 1e-12 on T <= 8."""
    rng = np.random.default_rng(18)
    for shape in (dict(B=1, H=4, G=2, d_h=8, d_n=6, d_r=2, lens=(8,)),
                  dict(B=3, H=8, G=2, d_h=6, d_n=6, d_r=4, lens=(3, 0, 7)),
                  dict(B=2, H=2, G=2, d_h=4, d_n=2, d_r=6, lens=(1, 5))):
        c = _rand_case(rng, extra=1, **shape)
        c["q_pos"] = c["q_pos"] + rng.integers(0, 50, size=len(c["q_pos"]))
        out, lse = orc.gva_decode(base=10000.0, **c)
        bo, bl = gva_decode_loops(c["q"], c["M"], c["q_pos"], c["V"], c["k_rope"], c["seq_offset"],
                                  c["seq_len"], c["d_n"], c["d_r"], 10000.0)
        assert np.max(np.abs(out - np.array(bo))) < 1e-12
        bl = np.array(bl)
        fin = np.isfinite(bl)
        assert np.array_equal(fin, np.isfinite(lse))
        assert np.max(np.abs(lse[fin] - bl[fin])) < 1e-12


def check_round_to_bf16(orc):
    """Values representable in float32 round exactly as torch's float32->bf16
    conversion (round to nearest, ties to even); exact halfway cases go to even."""
    rng = np.random.default_rng(19)
    x32 = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(orc.round_to_bf16(x32.astype(np.float64)), ref)
    one = 1.0
    ulp = 2.0 ** -7
    assert orc.round_to_bf16(np.array([one + ulp / 2]))[0] == one                 # tie -> even
    assert orc.round_to_bf16(np.array([one + 3 * ulp / 2]))[0] == one + 2 * ulp   # tie -> even
    assert orc.round_to_bf16(np.array([one + ulp / 2 + 2.0 ** -40]))[0] == one + ulp
    assert orc.round_to_bf16(np.array([-0.0, 0.0]))[1] == 0.0


def check_append(orc):
    rng = np.random.default_rng(20)
    S, G, d_h, d_r = 10, 2, 4, 6
    V0 = rng.standard_normal((S, G, d_h))
    K0 = rng.standard_normal((S, d_r))
    v = rng.standard_normal((3, G, d_h))
    k = rng.standard_normal((3, d_r))
    V1, K1, err = orc.append_cache(V0, K0, v, k, np.array([2, 9, 10]), np.array([5, 0, 1]), 10000.0, "f32")
    assert err == 1
    assert np.array_equal(V1[2], v[0]) and np.array_equal(V1[9], v[1])
    untouched = [i for i in range(S) if i not in (2, 9)]
    assert np.array_equal(V1[untouched], V0[untouched]) and np.array_equal(K1[untouched], K0[untouched])
    assert np.array_equal(K1[9], k[1].astype(np.float32).astype(np.float64))   # position 0: no rotation
    assert np.max(np.abs(K1[2] - orc.rope(k[0], 5.0, 10000.0))) < 1e-6         # float32 storage


def check_gqa_append(orc):
    """The GQA baseline's append: each group's key equals transformers' Llama rotary
    embedding over the full head width at the token's position (an implementation
    independent of the oracle's), rounded once to bf16; the value is copied; slots
    outside the cache are skipped and flagged."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    rng = np.random.default_rng(22)
    for d_h, G, base in ((8, 2, 10000.0), (64, 4, 10000.0), (128, 2, 500000.0)):
        S = 9
        K0 = orc.round_to_bf16(rng.standard_normal((S, G, d_h)))
        V0 = orc.round_to_bf16(rng.standard_normal((S, G, d_h)))
        k = orc.round_to_bf16(rng.standard_normal((4, G, d_h)))
        v = orc.round_to_bf16(rng.standard_normal((4, G, d_h)))
        slot, pos = np.array([3, 8, -1, 0]), np.array([0, 4093, 5, 77])
        K1, V1, err = orc.gqa_append_cache(K0, V0, k, v, slot, pos, base, "bf16")
        assert err == 1
        cfg = LlamaConfig(hidden_size=4 * d_h, num_attention_heads=4, head_dim=d_h, rope_theta=base)
        emb = LlamaRotaryEmbedding(cfg)
        for i in (0, 1, 3):
            xt = torch.from_numpy(k[i])[None, :, None, :]            # [1, G, 1, d_h]
            cos, sin = emb(xt, torch.tensor([[int(pos[i])]]))
            ref, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
            ref = ref[0, :, 0].numpy()
            s_ = slot[i]
            # transformers forms its angles in float32: compare before the bf16
            # rounding can amplify that, then check the stored value is a bf16
            assert np.max(np.abs(K1[s_] - ref)) <= 4e-3 * max(1.0, np.max(np.abs(ref))), (d_h, i)
            assert np.array_equal(orc.round_to_bf16(K1[s_]), K1[s_])
            assert np.array_equal(V1[s_], v[i])
        assert np.array_equal(K1[3], k[0])                           # position 0: unrotated
        untouched = [j for j in range(S) if j not in (3, 8, 0)]
        assert np.array_equal(K1[untouched], K0[untouched])
        assert np.array_equal(V1[untouched], V0[untouched])


def check_multi_query_causal(orc):
    """Several new tokens decoded together: one query reduces to the one-token
    decode; the last query sees the whole cache; query i does not see rows after
    its own position (changing them leaves it unchanged but moves later queries)."""
    rng = np.random.default_rng(21)
    c = _rand_case(rng, B=2, H=4, G=2, d_h=8, d_n=6, d_r=4, lens=(7, 5), extra=0)
    Q = 3
    q = rng.standard_normal((2, Q, 4, 10))
    qpos = np.stack([c["seq_len"] - Q + i for i in range(Q)], axis=1)
    args = dict(M=c["M"], V=c["V"], k_rope=c["k_rope"], seq_offset=c["seq_offset"],
                seq_len=c["seq_len"], d_n=6, d_r=4, base=10000.0)
    out, lse = orc.gva_decode_multi(q=q, q_pos=qpos, **args)
    one, one_l = orc.gva_decode_multi(q=q[:, :1], q_pos=c["seq_len"][:, None], **args)
    ref1, ref1_l = orc.gva_decode(q=q[:, 0], q_pos=c["seq_len"], **args)
    assert np.array_equal(one[:, 0], ref1) and np.array_equal(one_l[:, 0], ref1_l)
    last, last_l = orc.gva_decode(q=q[:, Q - 1], q_pos=qpos[:, Q - 1], **args)
    assert np.max(np.abs(out[:, Q - 1] - last)) < 1e-14
    V2 = c["V"].copy()
    for b in range(2):                         # change the last row of every sequence
        V2[c["seq_offset"][b] + c["seq_len"][b] - 1] += 1.0
    out2, _ = orc.gva_decode_multi(q=q, q_pos=qpos, **dict(args, V=V2))
    assert np.max(np.abs(out2[:, :Q - 1] - out[:, :Q - 1])) == 0
    assert np.max(np.abs(out2[:, Q - 1] - out[:, Q - 1])) > 1e-6


ALL_CHECKS = [check_cache_ratio, check_kv_shared_is_sdpa, check_gqa_is_sdpa, check_rope_matches_llama,
              check_relative_position, check_rope_group_law, check_absorption_identity,
              check_softmax_closed_forms, check_bruteforce, check_round_to_bf16, check_append,
              check_multi_query_causal, check_gqa_append]
