"""Decode with shared keys and values (K = V: M_h = I, d_r = 0) through its own
entry point, which reads the raw query: against the float64 oracle (the GQA
oracle with K = V, which the oracle pins show equals GVA with M = I);
bit-identical to the absorb route with an identity M on the same (mma.sync)
split kernel, and within rounding of the absorb route on the opt-in tcgen05
kernel."""
import numpy as np
import pytest
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import WORKLOADS, as_f64, make_decode_inputs
from gpu_helpers import assert_close, dev, lse_close, shape_of

pytestmark = pytest.mark.gpu


def shared_kv_workload(name):
    wl = WORKLOADS[name]
    return wl.scaled(name=name + "_kv", d_n=wl.d_h, d_r=0)


@pytest.mark.parametrize("name,lengths", [
    ("350m_b8_t4096", [4097, 1, 33, 0, 700, 64, 2, 1031]),
    ("d128_b1_t131072", [3000, 17]),
    ("ragged_b64_1k_16k", [16, 17, 1000]),
    ("tiny_fp32_t64", [64, 5]),
])
def test_shared_kv_matches_oracle_and_absorb_route(name, lengths):
    wl = shared_kv_workload(name)
    di = make_decode_inputs(wl, lengths=np.array(lengths))
    B = len(lengths)
    sh = shape_of(di)
    total = max(di.total_tokens, 1)
    q, V = dev(di.q), dev(di.V)
    soff, slen = dev(di.seq_offset), dev(di.seq_len)
    outs = []
    for route in ("shared", "absorb", "absorb-tcgen05"):
        sh = shape_of(di, flags=gva.FLAG_TCGEN05_PATH if route == "absorb-tcgen05" else 0)
        ws = gva.new_workspace(sh, total)
        out = torch.empty(B, wl.H, wl.d_h, device="cuda")
        lse = torch.empty(B, wl.H, device="cuda")
        if route == "shared":
            gva.shared_kv_decode_attention(sh, q, V, soff, slen, total, out, lse, ws)
        else:
            eye = torch.eye(wl.d_h, dtype=wl.torch_dtype).expand(wl.H, wl.d_h, wl.d_h).contiguous()
            q_abs = torch.empty(B, wl.H, wl.d_h, device="cuda")
            gva.absorb_query(sh, q, dev(eye), dev(di.q_pos), q_abs)
            kr = torch.zeros(1, 8, dtype=wl.torch_dtype, device="cuda")   # unused: d_r = 0
            gva.decode_attention(sh, q_abs, V, kr, soff, slen, total, out, lse, ws)
        torch.cuda.synchronize()
        assert gva.workspace_status(ws) == 0
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    ref, ref_lse = oracle.gqa_decode(as_f64(di.q), as_f64(di.V), as_f64(di.V), di.seq_offset.numpy(),
                                     di.seq_len.numpy())
    assert_close(outs[0][0], ref, wl.dtype, f"shared-kv {name}")
    lse_close(outs[0][1], ref_lse, f"shared-kv {name}")
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
    assert np.max(np.abs(outs[2][0] - outs[0][0])) < 1e-4
    a, b = outs[2][1], outs[0][1]
    assert np.array_equal(np.isneginf(a), np.isneginf(b))     # empty sequences: lse = -inf
    fin = np.isfinite(b)
    assert np.max(np.abs(a[fin] - b[fin]), initial=0.0) < 1e-4
