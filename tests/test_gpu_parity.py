"""CUDA path against the float64 oracle, element by element, through the C ABI.

Workloads are the five GVA decode shapes (reduced cache lengths here so the
oracle runs in seconds while still spanning many tiles and ragged tails; the
full sizes run in test_gpu_full_size.py on sampled outputs)."""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import (WORKLOADS, as_f64, make_append_inputs,
                                                make_decode_inputs, make_gqa_append_inputs,
                                                make_gqa_inputs)
from gpu_helpers import (LOG2E, assert_close, dev, lse_close, oracle_gqa, oracle_gva, run_gqa,
                         run_gva, shape_of)

pytestmark = pytest.mark.gpu

NAMES = list(WORKLOADS)


def small(name, lengths=None):
    """The workload with short caches: lengths that cross tile boundaries and
    leave ragged tails (tiles are 16, 32 or 64 rows)."""
    wl = WORKLOADS[name]
    if lengths is None:
        if wl.dtype == "f32":
            lengths = [64]
        else:
            base = [1, 15, 16, 17, 31, 33, 63, 65, 100, 257, 640, 1031]
            lengths = base[:max(2, min(len(base), wl.B + 4))]
    return make_decode_inputs(wl, extra_slots=1, lengths=np.array(lengths))


# ------------------------------------------------------------------ absorb

@pytest.mark.parametrize("name", NAMES)
def test_absorb_query(name):
    di = small(name)
    wl = di.wl
    _, _, q_abs, _ = run_gva(di)
    qt, qr = oracle.absorbed_query(as_f64(di.q), as_f64(di.M), di.q_pos.numpy(), wl.d_n, wl.d_r,
                                   wl.rope_base)
    c = LOG2E / math.sqrt(wl.d_n + wl.d_r)
    got_t = q_abs[:, :, :wl.d_h] / c
    got_r = q_abs[:, :, wl.d_h:] / c
    for got, ref in ((got_t, qt), (got_r, qr)):
        err = np.max(np.abs(got - ref)) / max(1.0, np.max(np.abs(ref)))
        assert err < 2e-6, err


# ------------------------------------------------------------------ append

@pytest.mark.parametrize("name", NAMES)
def test_append_cache(name):
    wl = WORKLOADS[name]
    di = make_decode_inputs(wl, extra_slots=2, lengths=np.array([5, 40, 3]))
    S = di.num_slots
    rng = np.random.default_rng(5)
    slots = rng.choice(S, size=24, replace=False).astype(np.int32)
    pos = rng.integers(0, 131072 * 2, size=24).astype(np.int32)
    slots[3] = S          # out of range: skipped, flagged
    slots[7] = -1
    ap = make_append_inputs(wl, slots, pos)
    V, KR = dev(di.V), dev(di.k_rope)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sh = shape_of(di)
    gva.append_cache(sh, dev(ap.v_new), dev(ap.kpe_new), dev(ap.slot), dev(ap.pos), V, KR, err)
    torch.cuda.synchronize()
    V_ref, K_ref, e_ref = oracle.append_cache(as_f64(di.V), as_f64(di.k_rope), as_f64(ap.v_new),
                                              as_f64(ap.kpe_new), slots, pos, wl.rope_base, wl.dtype)
    assert int(err.item()) == e_ref == 1
    # values: a bit-exact copy; untouched rows unchanged
    assert np.array_equal(as_f64(V.cpu()), V_ref)
    # rotated keys: both sides round the float64 rotation once to the cache type;
    # the only admissible difference is a tie decided differently by the last
    # float64 bit, which never happened on these draws
    got = as_f64(KR.cpu())
    same = got == K_ref
    assert same.all(), f"{(~same).sum()} rotated-key elements differ"


def test_append_then_decode_end_to_end():
    """Raw keys through the GPU append, then GPU decode, against the oracle's
    append followed by the oracle's decode."""
    wl = WORKLOADS["350m_b8_t4096"]
    lengths = np.array([70, 129, 1])
    di = make_decode_inputs(wl, extra_slots=1, lengths=lengths)
    V0, K0 = as_f64(di.V), as_f64(di.k_rope)
    offs = di.seq_offset.numpy()
    slots = (offs + lengths).astype(np.int32)
    ap = make_append_inputs(wl, slots, lengths.astype(np.int32))
    V, KR = dev(di.V), dev(di.k_rope)
    sh = shape_of(di)
    gva.append_cache(sh, dev(ap.v_new), dev(ap.kpe_new), dev(ap.slot), dev(ap.pos), V, KR)
    torch.cuda.synchronize()
    di.V, di.k_rope = V.cpu(), KR.cpu()
    di.seq_len = torch.from_numpy((lengths + 1).astype(np.int32))
    di.q_pos = di.seq_len.clone() - 1      # the new token queries at its own position
    out, lse, _, st = run_gva(di)
    V_ref, K_ref, _ = oracle.append_cache(V0, K0, as_f64(ap.v_new), as_f64(ap.kpe_new), slots, lengths,
                                          wl.rope_base, wl.dtype)
    ref, ref_lse = oracle.gva_decode(as_f64(di.q), as_f64(di.M), di.q_pos.numpy(), V_ref, K_ref,
                                     offs, di.seq_len.numpy(), wl.d_n, wl.d_r, wl.rope_base)
    assert st == 0
    assert_close(out, ref, wl.dtype, "append+decode")
    lse_close(lse, ref_lse)


@pytest.mark.parametrize("name", ["350m_b8_t4096", "dr24_b4_t32768"])
def test_append_then_decode_without_sync(name):
    """A decode requests its first cache tiles before its PDL wait; an append
    launched just before it on the stream lets it launch only once the new rows
    are stored.  Appended slots start out holding large garbage values, and each
    decode follows its append with no synchronisation in between."""
    wl = WORKLOADS[name]
    lengths = np.array([40, 3, 100, 1])      # short: the new row sits in a CTA's first tiles
    di = make_decode_inputs(wl, extra_slots=1, lengths=lengths)
    offs = di.seq_offset.numpy()
    slots = (offs + lengths).astype(np.int32)
    V0, KR0 = di.V.clone(), di.k_rope.clone()
    V0[torch.from_numpy(slots).long()] = 1000.0
    KR0[torch.from_numpy(slots).long()] = 1000.0
    ap = make_append_inputs(wl, slots, lengths.astype(np.int32))
    seq_len = torch.from_numpy((lengths + 1).astype(np.int32))
    q_pos = torch.from_numpy(lengths.astype(np.int32))
    B, total = len(lengths), int(seq_len.sum())
    sh = shape_of(di)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(q_pos), q_abs)
    soff, slen = dev(di.seq_offset), dev(seq_len)
    v_new, kpe_new, slot, pos = dev(ap.v_new), dev(ap.kpe_new), dev(ap.slot), dev(ap.pos)
    ws = gva.new_workspace(sh, total)
    pairs = []
    for _ in range(10):
        V, KR = dev(V0), dev(KR0)
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        gva.append_cache(sh, v_new, kpe_new, slot, pos, V, KR)
        gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out, lse, ws)
        pairs.append((out, lse))
    torch.cuda.synchronize()
    assert gva.workspace_status(ws) == 0
    V_ref, K_ref, _ = oracle.append_cache(as_f64(V0), as_f64(KR0), as_f64(ap.v_new),
                                          as_f64(ap.kpe_new), slots, lengths, wl.rope_base, wl.dtype)
    ref, ref_lse = oracle.gva_decode(as_f64(di.q), as_f64(di.M), q_pos.numpy(), V_ref, K_ref, offs,
                                     seq_len.numpy(), wl.d_n, wl.d_r, wl.rope_base)
    for out, lse in pairs:
        assert_close(out.cpu().numpy(), ref, wl.dtype, name)
        lse_close(lse.cpu().numpy(), ref_lse, name)


def test_absorb_then_decode_without_sync():
    """A plain decode reads its absorbed queries before its PDL wait; the absorb
    launched just before it lets it launch only once the queries are stored.
    Every iteration absorbs a different query into the same buffer (which held
    garbage first) and decodes at once, with no synchronisation."""
    wl = WORKLOADS["350m_b8_t4096"]
    di = small("350m_b8_t4096", lengths=[700, 33, 1500, 64])
    sh = shape_of(di)
    B, total = len(di.seq_len), di.total_tokens
    V, KR = dev(di.V), dev(di.k_rope)
    soff, slen, M, qpos = dev(di.seq_offset), dev(di.seq_len), dev(di.M), dev(di.q_pos)
    q_abs = torch.full((B, wl.H, wl.d_h + wl.d_r), 1e4, dtype=torch.float32, device="cuda")
    ws = gva.new_workspace(sh, total)
    rng = np.random.default_rng(21)
    qs, outs = [], []
    for _ in range(6):
        q = torch.from_numpy(rng.standard_normal(tuple(di.q.shape)).astype(np.float32)).to(di.q.dtype)
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        gva.absorb_query(sh, dev(q), M, qpos, q_abs)
        gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out, None, ws)
        qs.append(q)
        outs.append(out)
    torch.cuda.synchronize()
    assert gva.workspace_status(ws) == 0
    for q, out in zip(qs, outs):
        di.q = q
        ref, _ = oracle_gva(di)
        assert_close(out.cpu().numpy(), ref, wl.dtype, "absorb->decode")


def test_decode_step_then_decode_without_sync():
    """A fused step (its first kernel appends and absorbs, then the decode), then
    a plain decode of the same batch on the step's absorbed queries and updated
    cache, issued at once: the plain decode reads both before its own wait."""
    wl = WORKLOADS["350m_b8_t4096"]
    lengths = np.array([300, 65, 1, 1031])
    di = make_decode_inputs(wl, extra_slots=1, lengths=lengths)
    V0, K0 = as_f64(di.V), as_f64(di.k_rope)
    offs = di.seq_offset.numpy()
    slots = (offs + lengths).astype(np.int32)
    ap = make_append_inputs(wl, slots, lengths.astype(np.int32))
    seq_len = torch.from_numpy((lengths + 1).astype(np.int32))
    q_pos = torch.from_numpy(lengths.astype(np.int32))
    B, total = len(lengths), int(seq_len.sum())
    sh = shape_of(di)
    V, KR = dev(di.V), dev(di.k_rope)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    out1 = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    out2 = torch.empty_like(out1)
    ws1, ws2 = gva.new_workspace(sh, total), gva.new_workspace(sh, total)
    soff, slen = dev(di.seq_offset), dev(seq_len)
    gva.decode_step(sh, dev(di.q), dev(di.M), dev(q_pos), dev(ap.v_new), dev(ap.kpe_new),
                    dev(ap.slot), dev(ap.pos), V, KR, soff, slen, total, q_abs, out1, None, None, ws1)
    gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out2, None, ws2)
    torch.cuda.synchronize()
    assert gva.workspace_status(ws1) == 0 and gva.workspace_status(ws2) == 0
    V_ref, K_ref, _ = oracle.append_cache(V0, K0, as_f64(ap.v_new), as_f64(ap.kpe_new), slots, lengths,
                                          wl.rope_base, wl.dtype)
    ref, _ = oracle.gva_decode(as_f64(di.q), as_f64(di.M), q_pos.numpy(), V_ref, K_ref, offs,
                               seq_len.numpy(), wl.d_n, wl.d_r, wl.rope_base)
    assert_close(out1.cpu().numpy(), ref, wl.dtype, "step")
    assert_close(out2.cpu().numpy(), ref, wl.dtype, "decode after step")
    assert torch.equal(out1, out2)


def test_gqa_append_then_decode_without_sync():
    """The same for the GQA append and decode."""
    wl = WORKLOADS["350m_b8_t4096"]
    lengths = np.array([40, 3, 100, 1])
    gi = make_gqa_inputs(wl, extra_slots=1, lengths=lengths)
    offs = gi.seq_offset.numpy()
    slots = (offs + lengths).astype(np.int32)
    K0, V0 = gi.K.clone(), gi.V.clone()
    K0[torch.from_numpy(slots).long()] = 1000.0
    V0[torch.from_numpy(slots).long()] = 1000.0
    ap = make_gqa_append_inputs(wl, slots, lengths.astype(np.int32))
    seq_len = torch.from_numpy((lengths + 1).astype(np.int32))
    B, total = len(lengths), int(seq_len.sum())
    sh = gva.make_shape(B, wl.H, wl.G, wl.d_h, wl.d_h, 0, cache_dtype=wl.torch_dtype,
                        rope_base=wl.rope_base)
    q = dev(gi.q)
    soff, slen = dev(gi.seq_offset), dev(seq_len)
    ws = gva.new_workspace(sh, total)
    outs = []
    for _ in range(10):
        K, V = dev(K0), dev(V0)
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        gva.gqa_append_cache(sh, dev(ap.k_new), dev(ap.v_new), dev(ap.slot), dev(ap.pos), K, V)
        gva.gqa_decode_attention(sh, q, K, V, soff, slen, total, out, None, ws)
        outs.append((out, K))
    torch.cuda.synchronize()
    assert gva.workspace_status(ws) == 0
    K_ref, V_ref, _ = oracle.gqa_append_cache(as_f64(K0), as_f64(V0), as_f64(ap.k_new),
                                              as_f64(ap.v_new), slots, lengths, wl.rope_base,
                                              wl.dtype)
    from compressed_kv_cache_gva_b200.synth import GQAInputs
    ref, _ = oracle_gqa(GQAInputs(seq_len=seq_len, seq_offset=gi.seq_offset, q=gi.q,
                                  K=torch.from_numpy(K_ref), V=torch.from_numpy(V_ref),
                                  num_slots=gi.num_slots))
    for out, K in outs:
        assert np.array_equal(as_f64(K.cpu()), K_ref)
        assert_close(out.cpu().numpy(), ref, wl.dtype, "gqa")


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH, gva.FLAG_FMA_PATH],
                         ids=["tensor", "tcgen05", "fma"])
@pytest.mark.parametrize("name", NAMES)
def test_decode_matches_oracle(name, flags):
    di = small(name)
    out, lse, _, st = run_gva(di, flags=flags)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    assert_close(out, ref, di.wl.dtype, name)
    lse_close(lse, ref_lse, name)


def test_decode_fp32_ragged():
    di = small("tiny_fp32_t64", lengths=[64, 1, 17, 100, 0, 33])
    for flags in (0, gva.FLAG_FMA_PATH):
        out, lse, _, st = run_gva(di, flags=flags)
        ref, ref_lse = oracle_gva(di)
        assert st == 0
        assert_close(out, ref, "f32")
        lse_close(lse, ref_lse)


@pytest.mark.parametrize("cps", [1, 2, 3])
def test_decode_split_counts_agree(cps):
    """The split changes with CTAs per SM; the answer does not."""
    di = small("350m_b8_t4096", lengths=[4096, 777, 2048])
    out, lse, _, st = run_gva(di, ctas_per_sm=cps)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    assert_close(out, ref, "bf16", f"cps={cps}")


@pytest.mark.parametrize("lengths", [[0], [0, 0, 0], [1], [0, 5, 0, 1], [16, 0, 17], [33] * 9,
                                     [1] * 300], ids=["empty", "all-empty", "one", "mixed-empty",
                                                      "tile-edges", "many-small", "300x1"])
@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH], ids=["tensor", "tcgen05"])
def test_decode_edge_lengths(lengths, flags):
    di = small("350m_b8_t4096", lengths=lengths)
    out, lse, _, st = run_gva(di, flags=flags)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    L = np.array(lengths)
    assert np.all(out[L == 0] == 0)
    assert np.all(np.isneginf(lse[L == 0]))
    assert_close(out, ref, "bf16")
    lse_close(lse, ref_lse)


@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH], ids=["tensor", "tcgen05"])
@pytest.mark.parametrize("name", ["350m_b8_t4096", "dr24_b4_t32768", "d128_b1_t131072"])
def test_decode_growing_scores(name, flags):
    """Scores that jump far above everything before them inside one piece: the
    later rows' values are scaled up, so a row maximum grows by many units of
    log2 after the first tile (the kernels rescale their accumulated output then).
    Both orders, growing and shrinking, against the oracle."""
    di = small(name, lengths=[700, 1500, 90])
    wl = di.wl
    V = di.V.float().clone()
    offs = di.seq_offset.numpy()
    for b, L in enumerate(di.seq_len.numpy()):
        L = int(L)
        ramp = torch.linspace(0.2, 6.0, L) if b != 1 else torch.linspace(6.0, 0.2, L)
        V[offs[b]:offs[b] + L] *= ramp[:, None, None]
    di.V = V.to(di.V.dtype)
    out, lse, _, st = run_gva(di, flags=flags)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    assert_close(out, ref, wl.dtype, name)
    lse_close(lse, ref_lse, name)


@pytest.mark.parametrize("name", ["350m_b8_t4096", "dr24_b4_t32768", "ragged_b64_1k_16k",
                                  "d128_b1_t131072"])
def test_tcgen05_and_mma_sync_kernels_agree(name):
    """The two tensor-core split kernels (mma.sync, the default, and the opt-in
    tcgen05 one) compute the same decode; their outputs agree far inside the
    oracle bar."""
    di = small(name, lengths=[1, 31, 32, 33, 500, 4097, 16, 17][:max(3, min(8, di_b(name) + 3))])
    a, la, _, sa = run_gva(di)
    b, lb, _, sb = run_gva(di, flags=gva.FLAG_TCGEN05_PATH)
    assert sa == 0 and sb == 0
    assert np.max(np.abs(a - b)) < 2e-3
    assert np.max(np.abs(la - lb)) < 2e-3


def di_b(name):
    return WORKLOADS[name].B


def test_decode_length_one_returns_the_value_row():
    di = small("350m_b8_t4096", lengths=[1, 1])
    out, _, _, _ = run_gva(di)
    V = as_f64(di.V)
    for b in range(2):
        for h in range(16):
            np.testing.assert_allclose(out[b, h], V[di.seq_offset[b].item(), h // 4], rtol=0, atol=1e-6)


@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH], ids=["tensor", "tcgen05"])
def test_decode_large_batch_scan(flags):
    """4096 sequences exercise the in-kernel length scan over many threads, and
    CTAs that hold many short pieces."""
    rng = np.random.default_rng(3)
    lengths = rng.integers(0, 24, size=4096)
    di = small("350m_b8_t4096", lengths=lengths)
    pairs = [(b, h) for b in rng.choice(4096, 40, replace=False) for h in (0, 7, 15)]
    out, lse, _, st = run_gva(di, flags=flags)
    ref, ref_lse = oracle_gva(di, pairs=pairs)
    assert st == 0
    idx = tuple(np.array(pairs).T)
    assert_close(out[idx], ref[idx], "bf16")


def test_decode_bf16_output():
    di = small("350m_b8_t4096")
    out, _, _, _ = run_gva(di, out_dtype=torch.bfloat16)
    ref, _ = oracle_gva(di)
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH], ids=["tensor", "tcgen05"])
def test_decode_is_deterministic(flags):
    di = small("ragged_b64_1k_16k", lengths=[900, 3000, 17, 5000])
    outs = [run_gva(di, flags=flags)[0] for _ in range(5)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_decode_flags_slots_outside_cache():
    """A sequence that reaches past the cache is flagged in the status word;
    missing rows read as zeros and nothing faults."""
    di = small("350m_b8_t4096", lengths=[40, 40])
    di.seq_offset = torch.tensor([0, di.num_slots - 10], dtype=torch.int32)
    for flags in (0, gva.FLAG_FMA_PATH):
        out, _, _, st = run_gva(di, flags=flags)
        assert st & gva.DEVERR_RANGE
        assert np.all(np.isfinite(out))


# ------------------------------------------------------------------ GQA comparison kernel

@pytest.mark.parametrize("flags", [0, gva.FLAG_FMA_PATH], ids=["tensor", "fma"])
@pytest.mark.parametrize("name", ["350m_b8_t4096", "dr24_b4_t32768", "d128_b1_t131072"])
def test_gqa_matches_oracle(name, flags):
    wl = WORKLOADS[name]
    gi = make_gqa_inputs(wl, extra_slots=1, lengths=np.array([1, 33, 500, 1025]))
    out, lse, st = run_gqa(gi, wl.H, wl.G, wl.d_h, wl.torch_dtype, flags=flags)
    ref, ref_lse = oracle_gqa(gi)
    assert st == 0
    assert_close(out, ref, wl.dtype, name)
    lse_close(lse, ref_lse)


def test_shared_kv_gva_equals_gqa():
    """M_h = I and d_r = 0 turn GVA into attention with K = V: the GVA kernels
    and the GQA kernel (given K_cache = V_cache) agree with each other and with
    the oracle."""
    wl = WORKLOADS["350m_b8_t4096"].scaled(d_n=64, d_r=0)
    di = make_decode_inputs(wl, extra_slots=0, lengths=np.array([300, 1, 1000]))
    di.M = torch.eye(64, dtype=torch.bfloat16).expand(16, 64, 64).contiguous()
    out_gva, lse_gva, _, _ = run_gva(di)
    ref, ref_lse = oracle_gva(di)
    assert_close(out_gva, ref, "bf16", "gva K=V")
    # GQA with q = the absorbed query (identity map: q itself), K = V
    from compressed_kv_cache_gva_b200.synth import GQAInputs
    gi = GQAInputs(seq_len=di.seq_len, seq_offset=di.seq_offset, q=di.q, K=di.V, V=di.V,
                   num_slots=di.num_slots)
    out_gqa, lse_gqa, _ = run_gqa(gi, 16, 4, 64, torch.bfloat16)
    assert_close(out_gqa, ref, "bf16", "gqa K=V")
    assert np.max(np.abs(out_gqa - out_gva)) < 1e-3


# ------------------------------------------------------------------ fused decode step

@pytest.mark.parametrize("name,lengths", [
    ("350m_b8_t4096", [300, 65, 1, 1031]),
    ("d128_b1_t131072", [300, 65, 1, 1031]),
    ("d128_b1_t131072", [3000, 1500]),
    ("dr24_b4_t32768", [2000, 700, 5]),             # d_r = 24
    ("350m_b8_t4096", [4096] * 8),                  # the benchmark's batch shape
    ("tiny_fp32_t64", [300, 65, 1, 1031]),          # fp32 cache: CUDA-core path
])
def test_decode_step_matches_oracle_and_separate_calls(name, lengths):
    """gva_decode_step (append, absorb, decode in one call, decode streaming the
    cache before absorb finishes) against the oracle's append + decode, and
    bit-identical to the three separate calls."""
    wl = WORKLOADS[name]
    lengths = np.array(lengths)
    di = make_decode_inputs(wl, extra_slots=1, lengths=lengths)
    V0, K0 = as_f64(di.V), as_f64(di.k_rope)
    offs = di.seq_offset.numpy()
    slots = (offs + lengths).astype(np.int32)
    ap = make_append_inputs(wl, slots, lengths.astype(np.int32))
    seq_len = torch.from_numpy((lengths + 1).astype(np.int32))
    q_pos = torch.from_numpy(lengths.astype(np.int32))
    B = len(lengths)
    sh = shape_of(di)
    total = int(seq_len.sum())
    outs = []
    for fused in (True, False):
        V, KR = dev(di.V), dev(di.k_rope)
        q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda")
        ws = gva.new_workspace(sh, total)
        if fused:
            gva.decode_step(sh, dev(di.q), dev(di.M), dev(q_pos), dev(ap.v_new), dev(ap.kpe_new),
                            dev(ap.slot), dev(ap.pos), V, KR, dev(di.seq_offset), dev(seq_len), total,
                            q_abs, out, lse, None, ws)
        else:
            gva.append_cache(sh, dev(ap.v_new), dev(ap.kpe_new), dev(ap.slot), dev(ap.pos), V, KR)
            gva.absorb_query(sh, dev(di.q), dev(di.M), dev(q_pos), q_abs)
            gva.decode_attention(sh, q_abs, V, KR, dev(di.seq_offset), dev(seq_len), total, out, lse, ws)
        torch.cuda.synchronize()
        assert gva.workspace_status(ws) == 0
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    V_ref, K_ref, _ = oracle.append_cache(V0, K0, as_f64(ap.v_new), as_f64(ap.kpe_new), slots, lengths,
                                          wl.rope_base, wl.dtype)
    ref, ref_lse = oracle.gva_decode(as_f64(di.q), as_f64(di.M), q_pos.numpy(), V_ref, K_ref, offs,
                                     seq_len.numpy(), wl.d_n, wl.d_r, wl.rope_base)
    assert_close(outs[0][0], ref, wl.dtype, "decode_step")
    lse_close(outs[0][1], ref_lse)
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
