"""The same-shape GQA baseline's append and full decode step on the GPU, through
the C ABI, against the oracle: the append stores the value bit-exactly and each
group's key rotated over d_h and rounded once (onedev.kr review, "What differs":
GQA caches a key and a value per group and token); the step rotates the query,
appends and decodes, and equals the oracle's append followed by its GQA decode."""
import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import (WORKLOADS, as_f64, make_gqa_append_inputs,
                                                make_gqa_inputs)
from gpu_helpers import TOL, assert_close, dev, lse_close, rel_l2

pytestmark = pytest.mark.gpu


def gqa_shape(wl, B, **kw):
    return gva.make_shape(B, wl.H, wl.G, wl.d_h, wl.d_h, 0, cache_dtype=wl.torch_dtype,
                          rope_base=wl.rope_base, **kw)


@pytest.mark.parametrize("name", ["tiny_fp32_t64", "350m_b8_t4096", "d128_b1_t131072"])
def test_gqa_append_cache(name):
    wl = WORKLOADS[name]
    gi = make_gqa_inputs(wl, extra_slots=2, lengths=np.array([5, 40, 3]))
    S = gi.num_slots
    rng = np.random.default_rng(6)
    slots = rng.choice(S, size=20, replace=False).astype(np.int32)
    pos = rng.integers(0, 131072 * 2, size=20).astype(np.int32)
    slots[2] = S          # out of range: skipped, flagged
    slots[9] = -1
    ap = make_gqa_append_inputs(wl, slots, pos)
    K, V = dev(gi.K), dev(gi.V)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sh = gqa_shape(wl, 3)
    gva.gqa_append_cache(sh, dev(ap.k_new), dev(ap.v_new), dev(ap.slot), dev(ap.pos), K, V, err)
    torch.cuda.synchronize()
    K_ref, V_ref, e_ref = oracle.gqa_append_cache(as_f64(gi.K), as_f64(gi.V), as_f64(ap.k_new),
                                                  as_f64(ap.v_new), slots, pos, wl.rope_base,
                                                  wl.dtype)
    assert int(err.item()) == e_ref == 1
    assert np.array_equal(as_f64(V.cpu()), V_ref)          # bit-exact copy, others untouched
    # both sides round the float64 rotation once to the cache type
    same = as_f64(K.cpu()) == K_ref
    assert same.all(), f"{(~same).sum()} rotated key elements differ"


STEP_CASES = [("tiny_fp32_t64", [64, 17]), ("350m_b8_t4096", [4096, 77, 1, 0, 300]),
              ("dr24_b4_t32768", [2000, 31]), ("d128_b1_t131072", [5000])]


@pytest.mark.parametrize("name,lengths", STEP_CASES)
def test_gqa_decode_step_matches_oracle_and_separate_calls(name, lengths):
    """gqa_decode_step (query rotation + append in one kernel, decode streaming the
    cache behind it) against the oracle's rotation, append and GQA decode, and
    bit-identical to gqa_append_cache followed by gqa_decode_attention."""
    wl = WORKLOADS[name]
    L = np.array(lengths)
    B = len(L)
    gi = make_gqa_inputs(wl, extra_slots=1, lengths=L)
    offs = gi.seq_offset.numpy()
    slots = (offs + L).astype(np.int32)
    ap = make_gqa_append_inputs(wl, slots, L.astype(np.int32))
    seq_len = torch.from_numpy((L + 1).astype(np.int32))
    q_pos = torch.from_numpy(L.astype(np.int32))
    total = int(seq_len.sum())
    sh = gqa_shape(wl, B)
    res = []
    for fused in (True, False):
        K, V = dev(gi.K), dev(gi.V)
        q_rot = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda")
        ws = gva.new_workspace(sh, total)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if fused:
            gva.gqa_decode_step(sh, dev(gi.q), dev(q_pos), dev(ap.k_new), dev(ap.v_new),
                                dev(ap.slot), dev(ap.pos), K, V, dev(gi.seq_offset),
                                dev(seq_len), total, q_rot, out, lse, err, ws)
            q_rot_fused = q_rot.cpu().numpy()
        else:
            gva.gqa_append_cache(sh, dev(ap.k_new), dev(ap.v_new), dev(ap.slot), dev(ap.pos), K, V,
                                 err)
            sh_f = gqa_shape(wl, B, q_dtype=torch.float32)
            gva.gqa_decode_attention(sh_f, dev(torch.from_numpy(q_rot_fused)), K, V,
                                     dev(gi.seq_offset), dev(seq_len), total, out, lse, ws)
        torch.cuda.synchronize()
        assert gva.workspace_status(ws) == 0 and int(err.item()) == 0
        res.append((out.cpu().numpy(), lse.cpu().numpy()))
    q_ref = oracle.rope(as_f64(gi.q), q_pos.numpy()[:, None], wl.rope_base)
    assert rel_l2(q_rot_fused, q_ref) < 1e-6
    K_ref, V_ref, _ = oracle.gqa_append_cache(as_f64(gi.K), as_f64(gi.V), as_f64(ap.k_new),
                                              as_f64(ap.v_new), slots, L, wl.rope_base, wl.dtype)
    ref, ref_lse = oracle.gqa_decode(q_ref, K_ref, V_ref, offs, seq_len.numpy())
    assert_close(res[0][0], ref, wl.dtype, "gqa_decode_step")
    lse_close(res[0][1], ref_lse, "gqa_decode_step lse")
    assert np.array_equal(res[0][0], res[1][0]) and np.array_equal(res[0][1], res[1][1])
