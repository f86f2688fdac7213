"""Wide multi-token blocks (chunked prefill, long drafts: more than 8 query
columns per value group) on the tcgen05 kernel, through
gva_decode_attention_multi, against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import (WORKLOADS, as_f64, make_decode_inputs,
                                                make_multi_queries)
from gpu_helpers import assert_close, dev, lse_close, shape_of

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = [
    # (workload, n_query, lengths); rows per group = n_query * H/G, 128 per CTA
    (W["350m_b8_t4096"], 3, [700, 40, 3]),                  # 12 rows, ragged tiles
    (W["350m_b8_t4096"], 32, [1000, 32, 97]),               # 128 rows: one full block
    (W["350m_b8_t4096"], 40, [2049, 64, 41, 300]),          # 160 rows: two blocks
    (W["dr24_b4_t32768"], 24, [777, 130]),                  # d_r = 24 (32-wide positional tile)
    (W["d128_b1_t131072"], 16, [1500, 16]),                 # d_h = 128 (128-token tiles)
    (W["d128_b1_t131072"].scaled(name="d128r24", d_n=104, d_r=24), 40, [300, 129, 1]),
                                                            # d_h = 128, d_r = 24, two blocks
    (W["350m_b8_t4096"].scaled(name="kv", d_n=64, d_r=0), 33, [500, 66]),   # no positional slice
    (W["350m_b8_t4096"].scaled(name="mha", H=8, G=8), 64, [640, 64]),       # H/G = 1
    (W["350m_b8_t4096"], 5, [3, 0, 7]),                     # sequences shorter than the block
]


def run(wl, Q, lengths, out_dtype=torch.float32):
    lengths = np.asarray(lengths)
    di = make_decode_inputs(wl, lengths=lengths)
    B = len(lengths)
    q = make_multi_queries(wl, B, Q)
    qpos = torch.from_numpy(np.stack([lengths - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, wl.H, wl.d_h + wl.d_r, device="cuda")
    gva.absorb_query(sh_q, dev(q.reshape(B * Q, wl.H, -1)), dev(di.M), dev(qpos.reshape(-1)), q_abs)
    sh = shape_of(di, out_dtype=out_dtype)
    total = max(di.total_tokens, 1)
    n = gva.decode_workspace_size_multi(sh, Q, total)
    assert n > 0
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    out = torch.full((B, Q, wl.H, wl.d_h), float("nan"), dtype=out_dtype, device="cuda")
    lse = torch.full((B, Q, wl.H), float("nan"), device="cuda")
    kr = dev(di.k_rope) if wl.d_r else torch.zeros(1, 8, dtype=wl.torch_dtype, device="cuda")
    gva.decode_attention_multi(sh, Q, q_abs, dev(di.V), kr, dev(di.seq_offset), dev(di.seq_len),
                               total, out, lse, ws)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.gva_decode_multi(as_f64(q), as_f64(di.M), qpos.numpy(), as_f64(di.V),
                                           as_f64(di.k_rope), di.seq_offset.numpy(), lengths,
                                           wl.d_n, wl.d_r, wl.rope_base)
    return out.float().cpu().numpy(), lse.cpu().numpy(), ref, ref_lse, gva.workspace_status(ws)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_wide_multi_token_matches_oracle(case):
    wl, Q, lengths = CASES[case]
    out, lse, ref, ref_lse, st = run(wl, Q, lengths)
    assert st == 0
    assert_close(out, ref, wl.dtype, f"{wl.name} Q={Q}")
    lse_close(lse, ref_lse, f"{wl.name} Q={Q}")


def test_wide_multi_token_bf16_output():
    wl, Q, lengths = CASES[2]
    out, _, ref, _, st = run(wl, Q, lengths, out_dtype=torch.bfloat16)
    assert st == 0
    assert_close(out, ref, "bf16", "bf16 output")
