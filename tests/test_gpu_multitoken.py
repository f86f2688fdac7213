"""Decode of several new tokens per sequence at once (causal among them), as
used to verify drafted tokens in speculative decoding: CUDA path through the C
ABI against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, as_f64, make_decode_inputs, make_multi_queries
from gpu_helpers import assert_close, dev, lse_close, shape_of

pytestmark = pytest.mark.gpu


def run_multi(di, q, Q, out_dtype=torch.float32):
    """Absorb the B*Q query rows, then decode them causally.  Returns host
    (out [B,Q,H,d_h], lse [B,Q,H], workspace status)."""
    wl = di.wl
    B = len(di.seq_len)
    L = di.seq_len.numpy().astype(np.int64)
    qpos = torch.from_numpy(np.stack([L - Q + i for i in range(Q)], 1).astype(np.int32))
    sh_q = gva.make_shape(B * Q, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base)
    q_abs = torch.empty(B, Q, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh_q, dev(q.reshape(B * Q, wl.H, -1)), dev(di.M), dev(qpos.reshape(-1)), q_abs)
    sh = shape_of(di, out_dtype=out_dtype)
    total = max(di.total_tokens, 1)
    n = gva.decode_workspace_size_multi(sh, Q, total)
    assert n > 0
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    out = torch.empty(B, Q, wl.H, wl.d_h, dtype=out_dtype, device="cuda")
    lse = torch.empty(B, Q, wl.H, dtype=torch.float32, device="cuda")
    gva.decode_attention_multi(sh, Q, q_abs, dev(di.V), dev(di.k_rope), dev(di.seq_offset),
                               dev(di.seq_len), total, out, lse, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), gva.workspace_status(ws), qpos.numpy()


def oracle_multi(di, q, qpos):
    wl = di.wl
    return oracle.gva_decode_multi(as_f64(q), as_f64(di.M), qpos, as_f64(di.V), as_f64(di.k_rope),
                                   di.seq_offset.numpy(), di.seq_len.numpy(), wl.d_n, wl.d_r,
                                   wl.rope_base)


CASES = [
    # (workload, n_query, lengths): H/G * n_query columns per group, at most 8
    ("350m_b8_t4096", 2, [1500, 2, 3001, 17, 64, 65, 1, 700]),
    ("dr24_b4_t32768", 2, [4100, 33, 2]),
    ("d128_b1_t131072", 2, [2900, 130]),          # H/G = 4
    ("350m_b8_t4096", 1, [1500, 2, 3001]),
    ("mha_h8_g8", 4, [1000, 3, 4, 260]),          # H/G = 1: a thread's two columns are two queries
    ("h8_g4", 4, [777, 9]),                       # H/G = 2, 8 columns
    ("h8_g4", 2, [777, 9]),                       # H/G = 2, 4 columns
    ("mha_h8_g8", 3, [500, 2, 40]),               # 3 columns, one zero-query padding column
    ("h8_g4", 3, [777, 9, 64]),                   # 6 columns, two padding columns
]

EXTRA = {
    "mha_h8_g8": WORKLOADS["350m_b8_t4096"].scaled(name="mha_h8_g8", H=8, G=8),
    "h8_g4": WORKLOADS["350m_b8_t4096"].scaled(name="h8_g4", H=8, G=4),
}


@pytest.mark.parametrize("name,Q,lengths", CASES)
def test_multi_token_parity(name, Q, lengths):
    wl = EXTRA.get(name) or WORKLOADS[name]
    di = make_decode_inputs(wl, extra_slots=3, lengths=np.array(lengths))
    q = make_multi_queries(wl, len(lengths), Q)
    out, lse, st, qpos = run_multi(di, q, Q)
    assert st == 0
    ref, ref_lse = oracle_multi(di, q, qpos)
    assert_close(out, ref, wl.dtype, f"{name} Q={Q}")
    lse_close(lse, ref_lse, f"{name} Q={Q}")


def test_multi_token_q1_matches_single_decode():
    """One query token through the multi-token entry is the ordinary decode."""
    wl = WORKLOADS["350m_b8_t4096"]
    lengths = np.array([900, 5, 2049, 1])
    di = make_decode_inputs(wl, lengths=lengths)
    q = di.q.reshape(len(lengths), 1, wl.H, -1)
    out_m, lse_m, _, _ = run_multi(di, q, 1)
    sh = shape_of(di)
    q_abs = torch.empty(len(lengths), wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    qpos = dev(di.seq_len - 1)                 # the multi entry's new token is row L-1
    gva.absorb_query(sh, dev(di.q), dev(di.M), qpos, q_abs)
    ws = gva.new_workspace(sh, di.total_tokens)
    out = torch.empty(len(lengths), wl.H, wl.d_h, device="cuda")
    lse = torch.empty(len(lengths), wl.H, device="cuda")
    gva.decode_attention(sh, q_abs, dev(di.V), dev(di.k_rope), dev(di.seq_offset),
                         dev(di.seq_len), di.total_tokens, out, lse, ws)
    torch.cuda.synchronize()
    assert np.array_equal(out_m[:, 0], out.cpu().numpy())
    assert np.array_equal(lse_m[:, 0], lse.cpu().numpy())


def test_multi_token_shorter_than_queries():
    """A sequence holding fewer rows than new tokens: the first queries see
    nothing (zero output, lse = -inf)."""
    wl = WORKLOADS["350m_b8_t4096"]
    di = make_decode_inputs(wl, lengths=np.array([1, 0, 40]))
    q = make_multi_queries(wl, 3, 2)
    out, lse, st, qpos = run_multi(di, q, 2)
    ref, ref_lse = oracle_multi(di, q, qpos)
    assert st == 0
    assert_close(out, ref, wl.dtype, "short")
    lse_close(lse, ref_lse, "short")
    assert np.all(out[0, 0] == 0) and np.all(np.isneginf(lse[0, 0]))


def test_multi_token_unsupported_column_count():
    wl = WORKLOADS["350m_b8_t4096"].scaled(H=12)   # H/G = 3: 9 columns, 3 does not divide 128
    sh = gva.make_shape(1, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r)
    d = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt, device="cuda")
    ws = torch.zeros(max(gva.decode_workspace_size_multi(sh, 3, 64), 16), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(gva.GVAError):
        gva.decode_attention_multi(sh, 3, d(1, 3, wl.H, 80), d(64, wl.G, wl.d_h, dt=torch.bfloat16),
                                   d(64, wl.d_r, dt=torch.bfloat16),
                                   torch.zeros(1, dtype=torch.int32, device="cuda"),
                                   torch.full((1,), 64, dtype=torch.int32, device="cuda"), 64,
                                   d(1, 3, wl.H, wl.d_h), d(1, 3, wl.H), ws)
