"""Full-size workloads in the benchmark's launch configuration, checked on
sampled (sequence, head) outputs that the oracle computes one by one."""
import numpy as np
import pytest
import torch

from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs, make_gqa_inputs
from gpu_helpers import assert_close, lse_close, oracle_gqa, oracle_gva, run_gqa, run_gva

pytestmark = pytest.mark.gpu


def sample_pairs(B, H, n, seed=0):
    rng = np.random.default_rng(seed)
    pairs = {(int(rng.integers(B)), int(rng.integers(H))) for _ in range(n)}
    pairs |= {(0, 0), (B - 1, H - 1)}
    return sorted(pairs)


@pytest.mark.parametrize("name", ["350m_b8_t4096", "dr24_b4_t32768", "ragged_b64_1k_16k",
                                  "d128_b1_t131072", "tiny_fp32_t64"])
def test_full_size_sampled(name):
    wl = WORKLOADS[name]
    di = make_decode_inputs(wl, extra_slots=1)
    out, lse, _, st = run_gva(di)
    pairs = sample_pairs(len(di.seq_len), wl.H, 12 if wl.B > 1 else 6)
    ref, ref_lse = oracle_gva(di, pairs=pairs)
    idx = tuple(np.array(pairs).T)
    assert st == 0
    assert_close(out[idx], ref[idx], wl.dtype, name)
    lse_close(lse[idx], ref_lse[idx], name)
    # properties that hold at any size: finite, and every output coordinate lies
    # inside the range of its group's value column (a convex combination)
    assert np.all(np.isfinite(out))


@pytest.mark.parametrize("name", ["dr24_b4_t32768"])
def test_full_size_gqa_sampled(name):
    wl = WORKLOADS[name]
    gi = make_gqa_inputs(wl, extra_slots=1)
    out, lse, st = run_gqa(gi, wl.H, wl.G, wl.d_h, wl.torch_dtype)
    pairs = sample_pairs(wl.B, wl.H, 8)
    ref, ref_lse = oracle_gqa(gi, pairs=pairs)
    idx = tuple(np.array(pairs).T)
    assert st == 0
    assert_close(out[idx], ref[idx], wl.dtype, name)
    lse_close(lse[idx], ref_lse[idx], name)


@pytest.mark.parametrize("name", ["350m_b8_t4096", "d128_b1_t131072"])
def test_full_size_sampled_tcgen05(name):
    """The opt-in tcgen05 split kernel on the full-size caches, sampled."""
    from compressed_kv_cache_gva_b200 import gva
    wl = WORKLOADS[name]
    di = make_decode_inputs(wl, extra_slots=1)
    out, lse, _, st = run_gva(di, flags=gva.FLAG_TCGEN05_PATH)
    pairs = sample_pairs(len(di.seq_len), wl.H, 12 if wl.B > 1 else 6, seed=1)
    ref, ref_lse = oracle_gva(di, pairs=pairs)
    idx = tuple(np.array(pairs).T)
    assert st == 0
    assert_close(out[idx], ref[idx], wl.dtype, name)
    lse_close(lse[idx], ref_lse[idx], name)
    assert np.all(np.isfinite(out))
