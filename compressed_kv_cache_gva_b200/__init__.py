"""B200-native Grouped Value Attention (GVA) decode.

The hot path lives in hand-written CUDA kernels for sm_100a, exported through
the C ABI of ``libgva.so`` (include/gva.h).  ``gva`` is the thin ctypes binding;
``synth`` draws the seeded synthetic workloads used by the tests and benchmark.
"""
from . import gva  # noqa: F401  (the library itself loads on first call)
from .gva import (BF16, F32, FLAG_FMA_PATH, GVAError, Shape, absorb_query, append_cache,  # noqa: F401
                  decode_attention, decode_step, decode_workspace_size, gqa_decode_attention, make_shape,
                  new_workspace, workspace_status)
