"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare them."""
import math

import numpy as np
import torch

import oracle
from compressed_kv_cache_gva_b200 import gva
from compressed_kv_cache_gva_b200.synth import DecodeInputs, GQAInputs, as_f64

LOG2E = 1.4426950408889634

# Bars: bf16 caches -> max-abs <= 1e-2 and relative L2 <= 5e-3;
# float32 caches -> relative L2 <= 1e-5.
TOL = {"bf16": dict(max_abs=1e-2, rel_l2=5e-3), "f32": dict(max_abs=1e-4, rel_l2=1e-5)}


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    t = TOL[dtype]
    mx = float(np.max(np.abs(got - ref))) if got.size else 0.0
    r = rel_l2(got, ref)
    assert mx <= t["max_abs"] and r <= t["rel_l2"], f"{what}: max_abs={mx:.3e} rel_l2={r:.3e} ({dtype})"
    return mx, r


def shape_of(di: DecodeInputs, **kw):
    wl = di.wl
    return gva.make_shape(len(di.seq_len), wl.H, wl.G, wl.d_h, wl.d_n, wl.d_r,
                          cache_dtype=wl.torch_dtype, rope_base=wl.rope_base, **kw)


def dev(t):
    return t.to("cuda").contiguous()


def run_gva(di: DecodeInputs, flags=0, out_dtype=torch.float32, ctas_per_sm=0, want_lse=True,
            max_total=None):
    """absorb + decode on the GPU.  Returns (out, lse, q_abs, status word) on host."""
    sh = shape_of(di, out_dtype=out_dtype, flags=flags, ctas_per_sm=ctas_per_sm)
    wl = di.wl
    B = len(di.seq_len)
    q, M = dev(di.q), dev(di.M)
    qpos, soff, slen = dev(di.q_pos), dev(di.seq_offset), dev(di.seq_len)
    V, KR = dev(di.V), dev(di.k_rope)
    q_abs = torch.empty(B, wl.H, wl.d_h + wl.d_r, dtype=torch.float32, device="cuda")
    gva.absorb_query(sh, q, M, qpos, q_abs)
    total = di.total_tokens if max_total is None else max_total
    ws = gva.new_workspace(sh, total)
    out = torch.empty(B, wl.H, wl.d_h, dtype=out_dtype, device="cuda")
    lse = torch.empty(B, wl.H, dtype=torch.float32, device="cuda") if want_lse else None
    gva.decode_attention(sh, q_abs, V, KR, soff, slen, total, out, lse, ws)
    torch.cuda.synchronize()
    return (out.float().cpu().numpy(), None if lse is None else lse.cpu().numpy(),
            q_abs.cpu().numpy(), gva.workspace_status(ws))


def oracle_gva(di: DecodeInputs, pairs=None):
    wl = di.wl
    return oracle.gva_decode(as_f64(di.q), as_f64(di.M), di.q_pos.numpy(), as_f64(di.V),
                             as_f64(di.k_rope), di.seq_offset.numpy(), di.seq_len.numpy(),
                             wl.d_n, wl.d_r, wl.rope_base, pairs=pairs)


def run_gqa(gi: GQAInputs, H, G, d_h, dtype, flags=0, out_dtype=torch.float32):
    B = len(gi.seq_len)
    sh = gva.make_shape(B, H, G, d_h, d_h, 0, cache_dtype=dtype, out_dtype=out_dtype, flags=flags)
    total = int(gi.seq_len.sum())
    ws = gva.new_workspace(sh, total)
    out = torch.empty(B, H, d_h, dtype=out_dtype, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    gva.gqa_decode_attention(sh, dev(gi.q), dev(gi.K), dev(gi.V), dev(gi.seq_offset),
                             dev(gi.seq_len), total, out, lse, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), gva.workspace_status(ws)


def oracle_gqa(gi: GQAInputs, pairs=None):
    return oracle.gqa_decode(as_f64(gi.q), as_f64(gi.K), as_f64(gi.V), gi.seq_offset.numpy(),
                             gi.seq_len.numpy(), pairs=pairs)


def lse_close(got, ref, what=""):
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got)), f"{what}: lse finiteness differs"
    if fin.any():
        err = np.max(np.abs(got[fin] - ref[fin]))
        assert err < 2e-3, f"{what}: lse max err {err:.3e}"
    assert np.all(np.isneginf(got[~fin]))
