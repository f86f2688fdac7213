"""gva_decode_attention_noalloc, the decode for callers that cannot allocate.

Some callers have no way to get scratch memory: code running while a stream is
being captured into a CUDA graph (cudaMalloc is not allowed there), plug-ins
that only receive their input and output buffers from a framework whose caching
allocator owns the rest of device memory, and latency-critical paths that must
not call cudaMalloc because it can synchronise the device.  For them the library
keeps the split-KV scratch in a fixed array of its own device memory, and
gva_noalloc_status reads that scratch's device status word back.

These tests call that entry point through the C ABI and compare it with the
float64 oracle and with the regular entry point (caller-provided workspace) on
the same inputs, twice in a row with different batches, so that the second call
also shows that the shared scratch left over from the first call does not leak
into its result.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import assert_close, dev, lse_close, oracle_gva, shape_of

pytestmark = pytest.mark.gpu


def _both(di):
    """(out, lse) of the workspace entry point and of the no-alloc entry point,
    and the no-alloc call's device status word."""
    wl = di.wl
    sh = shape_of(di)
    B = len(di.seq_len)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    V, KR, soff, slen = dev(di.V), dev(di.k_rope), dev(di.seq_offset), dev(di.seq_len)
    total = di.total_tokens
    ws = gva.new_workspace(sh, total)
    outs, status = [], None
    for use_scratch in (False, True):
        out = torch.full((B, wl.H, wl.d_h), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        if use_scratch:
            gva.decode_attention_noalloc(sh, q_abs, V, KR, soff, slen, total, out, lse)
            status = gva.noalloc_status()
        else:
            gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out, lse, ws)
        torch.cuda.synchronize()
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    return outs, status


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls_in_a_row():
    rng = np.random.default_rng(23)
    batches = [
        make_decode_inputs(WORKLOADS["350m_b8_t4096"], extra_slots=1,
                           lengths=np.array([4096, 77, 1, 0, 3000])),
        make_decode_inputs(WORKLOADS["ragged_b64_1k_16k"], extra_slots=1,
                           lengths=rng.integers(1, 2500, size=12)),
    ]
    for di in batches:
        ((ref, ref_lse), (got, got_lse)), status = _both(di)
        assert status == 0
        orc, orc_lse = oracle_gva(di)
        assert_close(got, orc, di.wl.dtype, "no-alloc vs oracle")
        lse_close(got_lse, orc_lse, "no-alloc lse vs oracle")
        assert_close(got, ref, di.wl.dtype, "no-alloc vs workspace entry point")
        lse_close(got_lse, ref_lse, "no-alloc lse")


def test_noalloc_reports_device_errors_and_clears_them_on_the_next_call():
    """A sequence reaching past the cache sets GVA_DEVERR_RANGE in the scratch's
    status word, which gva_noalloc_status returns; the next valid call starts from
    a clear word.  (Rows past the cache read as zeros through the TMA bounds; the
    decode never addresses them.)"""
    di = make_decode_inputs(WORKLOADS["350m_b8_t4096"], extra_slots=1, lengths=np.array([40, 40]))
    sh = shape_of(di)
    wl = di.wl
    q_abs = torch.empty(2, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    V, KR, slen = dev(di.V), dev(di.k_rope), dev(di.seq_len)
    out = torch.empty(2, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    bad_off = torch.tensor([0, di.num_slots - 10], dtype=torch.int32, device="cuda")
    gva.decode_attention_noalloc(sh, q_abs, V, KR, bad_off, slen, 80, out)
    assert gva.noalloc_status() & gva.DEVERR_RANGE
    assert torch.isfinite(out).all()
    gva.decode_attention_noalloc(sh, q_abs, V, KR, dev(di.seq_offset), slen, 80, out)
    assert gva.noalloc_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch_without_touching_it():
    """A batch whose partials exceed the fixed scratch gets GVA_ERR_WORKSPACE and
    a message naming both sizes; nothing is launched, and the status word of the
    previous call is left as it was."""
    di = make_decode_inputs(WORKLOADS["350m_b8_t4096"], extra_slots=1, lengths=np.array([40, 40]))
    sh0 = shape_of(di)
    wl = di.wl
    q_abs = torch.empty(2, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh0, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    out = torch.empty(2, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    bad_off = torch.tensor([0, di.num_slots - 10], dtype=torch.int32, device="cuda")
    gva.decode_attention_noalloc(sh0, q_abs, dev(di.V), dev(di.k_rope), bad_off, dev(di.seq_len),
                                 80, out)
    assert gva.noalloc_status() & gva.DEVERR_RANGE

    sh = gva.make_shape(4096, 64, 8, 128, 112, 16)
    need = gva.decode_workspace_size(sh, 1 << 20)
    assert need > gva.NOALLOC_SCRATCH_BYTES
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    L = gva.lib()
    p = t.data_ptr()
    st = L.gva_decode_attention_noalloc(ctypes.byref(sh), p, p, p, p, p, 1 << 20, 1 << 20, p, None,
                                        None)
    assert st == 3
    msg = L.gva_last_error().decode()
    assert str(need) in msg and str(gva.NOALLOC_SCRATCH_BYTES) in msg
    # the rejected call did not clear the word the earlier call left
    assert gva.noalloc_status() & gva.DEVERR_RANGE
    # a NULL output pointer for the status is rejected on the host
    assert L.gva_noalloc_status(None, None) == 1
