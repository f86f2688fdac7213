"""bf16 caches with d_h = 32 on the tensor-core split kernel: a group's values
arrive as one 32-column box per tile with a 64-byte swizzle (64-wide groups use
128-byte boxes).  CUDA path through the C ABI against the float64 oracle: the GVA
decode at edge lengths, the same-shape GQA decode, a two-token decode, and a
full-length cache sampled pair by pair."""
import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import (WORKLOADS, as_f64, make_decode_inputs,
                                                make_gqa_inputs, make_multi_queries)
from gpu_helpers import (assert_close, dev, lse_close, oracle_gqa, oracle_gva, run_gqa, run_gva,
                         shape_of)

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny_fp32_t64"]
SHAPES = {
    "dh32_tiny_bf16": TINY.scaled(name="dh32_tiny_bf16", dtype="bf16"),            # H=4, G=2, d_r=8
    "dh32_h16_g4": TINY.scaled(name="dh32_h16_g4", dtype="bf16", B=8, H=16, G=4, T=4096),
    "dh32_h8_g8_dr24": TINY.scaled(name="dh32_h8_g8_dr24", dtype="bf16", H=8, G=8, d_n=8, d_r=24),
    "dh32_h8_g2": TINY.scaled(name="dh32_h8_g2", dtype="bf16", H=8, G=2),            # 4 heads per group
    "dh32_h16_g2": TINY.scaled(name="dh32_h16_g2", dtype="bf16", H=16, G=2),         # 8 heads per group
}


@pytest.mark.parametrize("lengths", [[0, 1, 63, 64, 65, 1000], [4097], [2]], ids=["edges", "long", "two"])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_dh32_decode_matches_oracle(name, lengths):
    wl = SHAPES[name]
    di = make_decode_inputs(wl, extra_slots=1, lengths=np.array(lengths))
    out, lse, _, st = run_gva(di)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    assert_close(out, ref, "bf16", name)
    lse_close(lse, ref_lse, name)


@pytest.mark.parametrize("name", ["dh32_tiny_bf16", "dh32_h16_g4"])
def test_dh32_gqa_matches_oracle(name):
    wl = SHAPES[name]
    gi = make_gqa_inputs(wl, extra_slots=1, lengths=np.array([1, 33, 500, 1025]))
    out, lse, st = run_gqa(gi, wl.H, wl.G, wl.d_h, wl.torch_dtype)
    ref, ref_lse = oracle_gqa(gi)
    assert st == 0
    assert_close(out, ref, "bf16", name)
    lse_close(lse, ref_lse, name)


def test_dh32_two_token_decode_matches_oracle():
    wl = SHAPES["dh32_tiny_bf16"]                      # H/G = 2: two tokens make 4 columns
    L = np.array([300, 2, 65])
    di = make_decode_inputs(wl, extra_slots=2, lengths=L)
    Q = 2
    B = len(L)
    q = make_multi_queries(wl, B, Q)
    qpos = torch.from_numpy(np.stack([L - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r, rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh_q, dev(q.reshape(B * Q, wl.H, -1)), dev(di.M), dev(qpos.reshape(-1)), q_abs)
    sh = shape_of(di)
    ws = torch.zeros(gva.decode_workspace_size_multi(sh, Q, di.total_tokens), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(B, Q, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    gva.decode_attention_multi(sh, Q, q_abs, dev(di.V), dev(di.k_rope), dev(di.seq_offset),
                               dev(di.seq_len), di.total_tokens, out, None, ws)
    torch.cuda.synchronize()
    assert gva.workspace_status(ws) == 0
    ref, _ = oracle.gva_decode_multi(as_f64(q), as_f64(di.M), qpos.numpy(), as_f64(di.V),
                                     as_f64(di.k_rope), di.seq_offset.numpy(), di.seq_len.numpy(),
                                     wl.d_n, wl.d_r, wl.rope_base)
    assert_close(out.cpu().numpy(), ref, "bf16", "dh32 two tokens")


def test_dh32_full_length_sampled():
    """8 sequences x 4096 tokens at H = 16, G = 4, d_h = 32, checked on sampled pairs."""
    wl = SHAPES["dh32_h16_g4"]
    di = make_decode_inputs(wl, extra_slots=1)
    out, lse, _, st = run_gva(di)
    rng = np.random.default_rng(5)
    pairs = sorted({(int(rng.integers(8)), int(rng.integers(16))) for _ in range(8)} | {(0, 0), (7, 15)})
    ref, ref_lse = oracle_gva(di, pairs=pairs)
    idx = tuple(np.array(pairs).T)
    assert st == 0
    assert_close(out[idx], ref[idx], "bf16", "dh32 full length")
    lse_close(lse[idx], ref_lse[idx], "dh32 full length")
    assert np.all(np.isfinite(out))
