"""Single-token decode with few query heads per value group (H/G = 1, 2, 3, and
5..7), on the tensor-core split kernel: such groups run the 4- or 8-column
configuration with zero-query padding columns that are never stored.  CUDA path
through the C ABI against the float64 oracle, at edge lengths (empty, one token,
tile edges, ragged tails) and on one full-size cache sampled pair by pair."""
import numpy as np
import pytest

from compressed_kv_cache_gva_b200.synth import WORKLOADS, make_decode_inputs
from gpu_helpers import assert_close, lse_close, oracle_gva, run_gva

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["350m_b8_t4096"]
SHAPES = {
    "hg1_d64": BASE.scaled(name="hg1_d64", H=4, G=4),
    "hg2_d64": BASE.scaled(name="hg2_d64", H=8, G=4),
    "hg3_d64": BASE.scaled(name="hg3_d64", H=12, G=4),
    "hg2_d64_dr24": WORKLOADS["dr24_b4_t32768"].scaled(name="hg2_d64_dr24", H=8, G=4),
    "hg6_d64_g2": BASE.scaled(name="hg6_d64_g2", H=12, G=2),
    "hg1_d128_g8": WORKLOADS["d128_b1_t131072"].scaled(name="hg1_d128_g8", H=8, G=8),
    "hg2_d128_g8": WORKLOADS["d128_b1_t131072"].scaled(name="hg2_d128_g8", H=16, G=8),
    "hg5_d128_g2": WORKLOADS["d128_b1_t131072"].scaled(name="hg5_d128_g2", H=10, G=2),
}
LENGTHS = [[0, 1, 31, 32, 33, 1000, 4097], [300, 7], [1]]


@pytest.mark.parametrize("lengths", LENGTHS, ids=["edges", "two", "one"])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_narrow_group_decode_matches_oracle(name, lengths):
    wl = SHAPES[name]
    di = make_decode_inputs(wl, extra_slots=1, lengths=np.array(lengths))
    out, lse, _, st = run_gva(di)
    ref, ref_lse = oracle_gva(di)
    assert st == 0
    assert_close(out, ref, wl.dtype, name)
    lse_close(lse, ref_lse, name)


@pytest.mark.parametrize("name", ["hg1_d128_g8", "hg2_d64"])
def test_narrow_group_full_size_sampled(name):
    """The full-length cache of the workload the shape derives from (131072 tokens
    for d_h = 128, 8 x 4096 for d_h = 64), checked on sampled (sequence, head) pairs."""
    wl = SHAPES[name]
    di = make_decode_inputs(wl, extra_slots=1)
    out, lse, _, st = run_gva(di)
    rng = np.random.default_rng(4)
    B = len(di.seq_len)
    pairs = sorted({(int(rng.integers(B)), int(rng.integers(wl.H))) for _ in range(8)}
                   | {(0, 0), (B - 1, wl.H - 1)})
    ref, ref_lse = oracle_gva(di, pairs=pairs)
    idx = tuple(np.array(pairs).T)
    assert st == 0
    assert_close(out[idx], ref[idx], wl.dtype, name)
    lse_close(lse[idx], ref_lse[idx], name)
    assert np.all(np.isfinite(out))
