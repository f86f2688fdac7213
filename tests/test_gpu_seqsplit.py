"""A batch whose sequences are split into R parts (one part per GPU in the
multi-GPU layout), decoded part by part and merged with gva_merge_states, on one
GPU, against the float64 oracle on the whole cache."""
import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import gva, seqsplit
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import assert_close, dev, lse_close, oracle_gva, shape_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R", [1, 2, 3, 4])
@pytest.mark.parametrize("name", ["dr24_b4_t32768", "d128_b1_t131072", "350m_b8_t4096"])
def test_split_decode_and_merge(name, R):
    wl = WORKLOADS[name]
    lengths = np.array([2, 700, 3001, 1][:wl.B + 3])        # some parts empty when L < R
    di = make_decode_inputs(wl, extra_slots=0, lengths=lengths)
    sh = shape_of(di)
    B = len(lengths)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    merger = seqsplit.SequenceSplitMerge(sh, R, "cuda")
    for r in range(R):
        V_r, K_r, off_r, len_r, _ = seqsplit.shard_cache(dev(di.V), dev(di.k_rope), di.seq_offset,
                                                         di.seq_len, R, r)
        tot = int(len_r.sum())
        ws = gva.new_workspace(sh, max(tot, 1))
        gva.decode_attention(sh, q_abs, V_r, K_r, dev(off_r), dev(len_r), tot, merger.outs[r],
                             merger.lses[r], ws)
    out = torch.empty(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda")
    gva.merge_states(sh, merger.outs, merger.lses, out, lse)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_gva(di)
    assert_close(out.cpu().numpy(), ref, wl.dtype, f"{name} R={R}")
    lse_close(lse.cpu().numpy(), ref_lse)


def test_merge_all_empty_parts():
    sh = gva.make_shape(2, 4, 2, 64, 48, 16)
    outs = torch.randn(3, 2, 4, 64, device="cuda")
    lses = torch.full((3, 2, 4), float("-inf"), device="cuda")
    lses[1, 1] = 0.5                      # sequence 1: only part 1 is non-empty
    out = torch.empty(2, 4, 64, device="cuda")
    lse = torch.empty(2, 4, device="cuda")
    gva.merge_states(sh, outs, lses, out, lse)
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.allclose(out[1], outs[1, 1]) and torch.allclose(lse[1], lses[1, 1])
