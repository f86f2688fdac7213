"""gva_decode_step with its per-step inputs (query, new value, new positional key,
slot, position) in page-locked host memory and its output written into page-locked
host memory: with unified addressing the kernels access those buffers directly,
with no copy.  The result must be bit-identical to the same step on device buffers,
and the cache rows the step appends must be the same."""
import ctypes

import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_append_inputs, make_decode_inputs
from gpu_helpers import dev, shape_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,lengths", [("350m_b8_t4096", [4096, 77, 1, 0, 300]),
                                          ("d128_b1_t131072", [2000])])
def test_step_on_pinned_host_buffers_matches_device_buffers(name, lengths):
    wl = WORKLOADS[name]
    L = np.array(lengths)
    B = len(L)
    di = make_decode_inputs(wl, extra_slots=1, lengths=L)
    slots = (di.seq_offset.numpy() + L).astype(np.int32)
    ap = make_append_inputs(wl, slots, L.astype(np.int32))
    sh = shape_of(di)
    seq_len = dev(torch.from_numpy((L + 1).astype(np.int32)))
    total = int(L.sum()) + B
    inputs = [di.q, ap.v_new, ap.kpe_new, ap.slot, ap.pos]
    res = []
    for pinned in (False, True):
        V, KR = dev(di.V), dev(di.k_rope)
        q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
        ws = gva.new_workspace(sh, total)
        if pinned:
            q, v_new, kpe_new, slot, pos = (t.contiguous().pin_memory() for t in inputs)
            out = torch.full((B, wl.H, wl.d_h), float("nan"), dtype=torch.float32).pin_memory()
        else:
            q, v_new, kpe_new, slot, pos = (dev(t) for t in inputs)
            out = torch.full((B, wl.H, wl.d_h), float("nan"), dtype=torch.float32, device="cuda")
        rc = gva.lib().gva_decode_step(
            ctypes.byref(sh), q.data_ptr(), dev(di.M).data_ptr(), dev(di.q_pos).data_ptr(), B,
            v_new.data_ptr(), kpe_new.data_ptr(), slot.data_ptr(), pos.data_ptr(), V.data_ptr(),
            KR.data_ptr(), V.shape[0], dev(di.seq_offset).data_ptr(), seq_len.data_ptr(), total,
            q_abs.data_ptr(), out.data_ptr(), None, None, ws.data_ptr(), ws.numel(),
            torch.cuda.current_stream().cuda_stream)
        assert rc == 0, gva.lib().gva_last_error()
        torch.cuda.synchronize()
        assert gva.workspace_status(ws) == 0
        res.append((out.cpu().numpy(), V.cpu(), KR.cpu()))
    assert np.all(np.isfinite(res[1][0]))
    assert np.array_equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1], res[1][1]) and torch.equal(res[0][2], res[1][2])
