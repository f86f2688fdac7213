"""gva_decode_attention_noalloc, the decode for callers that cannot allocate.

Some callers have no way to get scratch memory: code running while a stream is
being captured into a CUDA graph (cudaMalloc is not allowed there), plug-ins
that only receive their input and output buffers from a framework whose caching
allocator owns the rest of device memory, and latency-critical paths that must
not call cudaMalloc because it can synchronise the device.  For them the library
keeps the split-KV scratch in a fixed array of its own device memory.

These tests call that entry point through the C ABI and compare it with the
regular entry point (caller-provided workspace) on the same inputs, twice in a
row with different batches, so that the second call also shows that the shared
scratch left over from the first call does not leak into its result.  This file
is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import assert_close, dev, lse_close, shape_of

pytestmark = pytest.mark.gpu


def _both(di):
    """(out, lse) of the workspace entry point and of the no-alloc entry point."""
    wl = di.wl
    sh = shape_of(di)
    B = len(di.seq_len)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    V, KR, soff, slen = dev(di.V), dev(di.k_rope), dev(di.seq_offset), dev(di.seq_len)
    total = di.total_tokens
    ws = gva.new_workspace(sh, total)
    outs = []
    for use_scratch in (False, True):
        out = torch.full((B, wl.H, wl.d_h), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        if use_scratch:
            gva.decode_attention_noalloc(sh, q_abs, V, KR, soff, slen, total, out, lse)
        else:
            gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out, lse, ws)
        torch.cuda.synchronize()
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    return outs


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    rng = np.random.default_rng(23)
    batches = [
        make_decode_inputs(WORKLOADS["350m_b8_t4096"], extra_slots=1,
                           lengths=np.array([4096, 77, 1, 0, 3000])),
        make_decode_inputs(WORKLOADS["ragged_b64_1k_16k"], extra_slots=1,
                           lengths=rng.integers(1, 2500, size=12)),
    ]
    for di in batches:
        (ref, ref_lse), (got, got_lse) = _both(di)
        assert_close(got, ref, di.wl.dtype, "no-alloc vs workspace entry point")
        lse_close(got_lse, ref_lse, "no-alloc lse")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """A batch whose partials exceed the fixed scratch gets GVA_ERR_WORKSPACE and
    a message naming both sizes; nothing is launched."""
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
