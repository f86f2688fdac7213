"""The C ABI library: it builds, loads, exports every symbol the header
declares, and validates arguments on the host (CPU only, no kernel runs)."""
import ctypes
import os
import re

import pytest

from compressed_kv_cache_gva_b200 import _build, gva

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gva.h")


@pytest.fixture(scope="module")
def L():
    _build.build()
    return gva.lib()


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("gva_absorb_query", "gva_append_cache", "gva_decode_attention",
              "gqa_decode_attention", "gva_decode_workspace_size", "gva_status_string",
              "gva_last_error"):
        assert n in names, n


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), f"{n} declared in gva.h but not exported"
    assert sorted(gva.EXPORTS) == declared_functions()


def test_shape_struct_layout():
    # gva_shape_t: 10 x 4-byte fields, a double at offset 40, float + int32 after it
    assert ctypes.sizeof(gva.Shape) == 56
    assert gva.Shape.rope_base.offset == 40
    assert gva.Shape.softmax_scale.offset == 48


def test_status_strings(L):
    for code, text in [(0, b"ok"), (1, b"invalid argument"), (2, b"unsupported shape"),
                       (3, b"workspace too small"), (4, b"CUDA error")]:
        assert L.gva_status_string(code) == text


def _shape(**kw):
    base = dict(B=2, H=16, G=4, d_h=64, d_n=48, d_r=16)
    base.update(kw)
    return gva.make_shape(**base)


FAKE = 1 << 20    # never dereferenced: validation rejects before any CUDA call


@pytest.mark.parametrize("bad", [dict(H=15), dict(G=0), dict(d_r=15), dict(d_h=0), dict(B=-1),
                                 dict(B=5000), dict(d_r=-2), dict(rope_base=0.0),
                                 dict(softmax_scale=-1.0), dict(ctas_per_sm=99)])
def test_invalid_shapes_are_rejected(L, bad):
    sh = _shape(**bad)
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 100, FAKE, None,
                                FAKE, 1 << 20, None)
    assert st == 1
    assert L.gva_last_error()
    assert L.gva_decode_workspace_size(ctypes.byref(sh), 100) == 0 or bad.keys() <= {"d_r", "rope_base"}


def test_null_and_misaligned_pointers(L):
    sh = _shape()
    st = L.gva_decode_attention(ctypes.byref(sh), None, FAKE, FAKE, FAKE, FAKE, 100, 100, FAKE, None,
                                FAKE, 1 << 20, None)
    assert st == 1 and b"NULL" in L.gva_last_error()
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE + 4, FAKE, FAKE, FAKE, FAKE, 100, 100, FAKE,
                                None, FAKE, 1 << 20, None)
    assert st == 1 and b"aligned" in L.gva_last_error()
    st = L.gva_absorb_query(ctypes.byref(sh), FAKE, FAKE + 8, FAKE, FAKE, None)
    assert st == 1
    st = L.gva_append_cache(ctypes.byref(sh), 4, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, None, None)
    assert st == 1 and b"num_slots" in L.gva_last_error()
    st = L.gva_append_cache(ctypes.byref(sh), -1, FAKE, FAKE, FAKE, FAKE, 10, FAKE, FAKE, None, None)
    assert st == 1


def test_bad_sizes(L):
    sh = _shape()
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 0, FAKE, None,
                                FAKE, 1 << 20, None)
    assert st == 1 and b"num_slots" in L.gva_last_error()
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 31, 100, FAKE,
                                None, FAKE, 1 << 20, None)
    assert st == 1 and b"max_total_tokens" in L.gva_last_error()
    sh = _shape(G=3, H=12, d_h=40, d_r=6)      # rows of 240 B ok, k_rope rows of 12 B are not
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 100, FAKE, None,
                                FAKE, 1 << 20, None)
    assert st == 1 and b"16 bytes" in L.gva_last_error()


def test_empty_batch_and_empty_append_are_noops(L):
    sh = _shape(B=0)
    assert L.gva_decode_attention(ctypes.byref(sh), None, None, None, None, None, 0, 1, None, None,
                                  None, 0, None) == 0
    sh = _shape()
    assert L.gva_append_cache(ctypes.byref(sh), 0, None, None, None, None, 1, None, None, None,
                              None) == 0


def test_no_device_is_a_cuda_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    sh = _shape()
    st = L.gva_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 100, FAKE, None,
                                FAKE, 1 << 20, None)
    assert st == 4


def test_shared_kv_needs_keys_equal_to_values(L):
    """The shared-KV entry takes only shapes where the keys are the values:
    no positional slice and a content width equal to the value width."""
    for bad in (dict(d_r=16), dict(d_n=48, d_r=0)):
        sh = _shape(**bad)
        st = L.gva_shared_kv_decode_attention(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, 100, 100,
                                              FAKE, None, FAKE, 1 << 20, None)
        assert st == 1 and b"shared keys and values" in L.gva_last_error()


def test_gqa_append_and_step_validate_on_the_host(L):
    """The GQA baseline's append and step reject, before any launch, a head width
    its RoPE cannot rotate (odd or above 128), a non-positive RoPE base, NULL
    pointers and misaligned ones; N = 0 appends nothing."""
    for bad, code in ((dict(d_h=130, d_n=130, d_r=0), 2), (dict(d_h=72, d_n=72, d_r=0, G=2, H=8), 0),
                      (dict(d_h=64, d_n=64, d_r=0, rope_base=-1.0), 1)):
        sh = _shape(**bad)
        st = L.gqa_append_cache(ctypes.byref(sh), 4, FAKE, FAKE, FAKE, FAKE, 10, FAKE, FAKE, None,
                                None)
        if code == 0:      # a valid shape: only the fake pointers stop it (no device here)
            continue
        assert st == code, (bad, st)
    sh = _shape(d_h=64, d_n=64, d_r=0)
    st = L.gqa_append_cache(ctypes.byref(sh), 4, None, FAKE, FAKE, FAKE, 10, FAKE, FAKE, None, None)
    assert st == 1 and b"NULL" in L.gva_last_error()
    st = L.gqa_append_cache(ctypes.byref(sh), 4, FAKE + 2, FAKE, FAKE, FAKE, 10, FAKE, FAKE, None,
                            None)
    assert st == 1 and b"aligned" in L.gva_last_error()
    assert L.gqa_append_cache(ctypes.byref(sh), 0, None, None, None, None, 1, None, None, None,
                              None) == 0
    st = L.gqa_decode_step(ctypes.byref(sh), FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10,
                           FAKE, FAKE, 100, None, FAKE, None, None, FAKE, 1 << 20, None)
    assert st == 1 and b"NULL" in L.gva_last_error()


def test_steps_check_the_decode_before_launching(L):
    """gva_decode_step and gqa_decode_step run every check of their decode (pointers,
    alignment, sizes) before their first kernel: a misaligned output or a bad cache
    size is an INVALID_ARG status, not a launch followed by an error."""
    sh = _shape()
    st = L.gva_decode_step(ctypes.byref(sh), FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           100, FAKE, FAKE, 100, FAKE, FAKE + 4, None, None, FAKE, 1 << 20, None)
    assert st == 1 and b"aligned" in L.gva_last_error()
    st = L.gva_decode_step(ctypes.byref(sh), FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           0, FAKE, FAKE, 100, FAKE, FAKE, None, None, FAKE, 1 << 20, None)
    assert st == 1 and b"num_slots" in L.gva_last_error()
    shg = _shape(d_h=64, d_n=64, d_r=0)
    st = L.gqa_decode_step(ctypes.byref(shg), FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100,
                           FAKE, FAKE, 100, FAKE, FAKE + 8, None, None, FAKE, 1 << 20, None)
    assert st == 1 and b"aligned" in L.gva_last_error()
    st = L.gqa_decode_step(ctypes.byref(shg), FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100,
                           FAKE, FAKE, 1 << 31, FAKE, FAKE, None, None, FAKE, 1 << 20, None)
    assert st == 1 and b"max_total_tokens" in L.gva_last_error()


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: without the compiled library the binding raises on first use."""
    import subprocess
    import sys
    code = ("from compressed_kv_cache_gva_b200 import gva\n"
            f"gva.LIB_PATH = {str(tmp_path / 'libgva.so')!r}\n"
            "gva.lib()\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "is missing" in r.stderr
