"""Reuse of one decode workspace across calls of different batches (a serving
loop whose batch changes every step): results equal those of fresh workspaces
and the status word stays 0."""
import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import dev, shape_of

pytestmark = pytest.mark.gpu


def _decode(di, ws):
    wl = di.wl
    B = len(di.seq_len)
    sh = shape_of(di)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    out = torch.empty(B, wl.H, wl.d_h, device="cuda")
    lse = torch.empty(B, wl.H, device="cuda")
    gva.decode_attention(sh, q_abs, dev(di.V), dev(di.k_rope), dev(di.seq_offset),
                         dev(di.seq_len), max(di.total_tokens, 1), out, lse, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name", ["350m_b8_t4096", "d128_b1_t131072"])
def test_workspace_reused_across_batches(name):
    wl = WORKLOADS[name]
    batches = [[700, 1, 3000], [5, 9000, 17, 64, 0, 2], [4097] * 8, [1]]
    big = max(gva.decode_workspace_size(
        gva.make_shape(len(L), wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r), 9100 * 8) for L in batches)
    shared = torch.zeros(big, dtype=torch.uint8, device="cuda")
    for lengths in batches * 2:
        di = make_decode_inputs(wl, lengths=np.array(lengths))
        got = _decode(di, shared)
        fresh = _decode(di, gva.new_workspace(shape_of(di), max(di.total_tokens, 1)))
        assert np.array_equal(got[0], fresh[0]) and np.array_equal(got[1], fresh[1])
        assert gva.workspace_status(shared) == 0


def _decode_flags(di, ws, max_total, flags):
    wl = di.wl
    B = len(di.seq_len)
    sh = shape_of(di, flags=flags)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    out = torch.empty(B, wl.H, wl.d_h, device="cuda")
    lse = torch.empty(B, wl.H, device="cuda")
    gva.decode_attention(sh, q_abs, dev(di.V), dev(di.k_rope), dev(di.seq_offset),
                         dev(di.seq_len), max_total, out, lse, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("flags", [0, gva.FLAG_TCGEN05_PATH, gva.FLAG_FMA_PATH],
                         ids=["tensor", "tcgen05", "fma"])
@pytest.mark.parametrize("name", ["350m_b8_t4096", "d128_b1_t131072"])
def test_token_bound_far_above_the_batch(name, flags):
    """max_total_tokens is an upper bound: a small batch decoded with a bound sized for
    capacity has fewer tiles than the grid has CTAs.  The batch runs in a workspace whose
    partial slots a larger batch filled just before, so a slot read but not rewritten
    would corrupt the result."""
    from gpu_helpers import assert_close, lse_close, oracle_gva
    wl = WORKLOADS[name]
    bound = 300_000
    shared = torch.zeros(gva.decode_workspace_size(
        gva.make_shape(70, wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r, flags=flags), bound),
        dtype=torch.uint8, device="cuda")
    big = make_decode_inputs(wl, lengths=np.array([4097] * 8))
    _decode_flags(big, shared, big.total_tokens, flags)
    for lengths in ([5, 40, 100, 0, 1], [3] * 70, [33]):
        di = make_decode_inputs(wl, lengths=np.array(lengths))
        out, lse = _decode_flags(di, shared, bound, flags)
        ref, ref_lse = oracle_gva(di)
        assert gva.workspace_status(shared) == 0
        assert_close(out, ref, wl.dtype, f"{name} {lengths[:5]}")
        lse_close(lse, ref_lse, f"{name} {lengths[:5]}")
        _decode_flags(big, shared, big.total_tokens, flags)   # refill the slots
