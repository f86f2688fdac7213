"""Failure detection without a GPU fault: a bounded pipeline wait that runs out.

The library's mbarrier waits give up after a poll and wall-time limit, set
GVA_DEVERR_WAIT in the workspace's status word, drain the copies they issued and
return, so a stuck pipeline ends the call instead of hanging the GPU.  A
test-only build of the library (libgva_waittest.so: 50 ms wait limit, and the
split kernel's producer never requests the second tile of each CTA, so no copy
is ever in flight for it) makes the consumers' wait on that tile run out.  The
call must return, report GVA_DEVERR_WAIT, and leave the context usable: the
regular library then decodes the same inputs correctly in the same process."""
import ctypes
import time

import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200 import _build, gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import assert_close, dev, oracle_gva, shape_of, run_gva

pytestmark = pytest.mark.gpu


def test_withheld_tile_makes_the_bounded_wait_report_and_return():
    _build.build_wait_test()
    L = gva.load(_build.WAIT_TEST_LIB)
    wl = WORKLOADS["350m_b8_t4096"]
    # 2 x 16384 tokens: ~1024 tiles over the grid, several per CTA, so every CTA
    # reaches its withheld second tile
    di = make_decode_inputs(wl, extra_slots=1, lengths=np.array([16384, 16384]))
    sh = shape_of(di)
    B = 2
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, dev(di.q), dev(di.M), dev(di.q_pos), q_abs)
    V, KR, soff, slen = dev(di.V), dev(di.k_rope), dev(di.seq_offset), dev(di.seq_len)
    total = di.total_tokens
    ws = gva.new_workspace(sh, total)
    out = torch.zeros(B, wl.H, wl.d_h, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.time()
    st = L.gva_decode_attention(ctypes.byref(sh), q_abs.data_ptr(), V.data_ptr(), KR.data_ptr(),
                                soff.data_ptr(), slen.data_ptr(), total, V.shape[0],
                                out.data_ptr(), None, ws.data_ptr(), ws.numel(), stream)
    assert st == 0, L.gva_last_error()
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert gva.workspace_status(ws) & gva.DEVERR_WAIT
    assert elapsed < 30, f"the bounded waits took {elapsed:.1f} s"
    # the context is still usable: the regular library decodes the same inputs
    got, _, _, status = run_gva(di)
    assert status == 0
    assert_close(got, oracle_gva(di)[0], wl.dtype, "decode after a wait timeout")
