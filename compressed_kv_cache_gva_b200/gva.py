"""Thin Python binding of libgva.so (argument marshalling only).

Every function takes torch tensors that already live on the current CUDA
device, passes their raw pointers and the current stream to the C ABI declared
in include/gva.h, and raises GVAError on a non-OK status.  All arithmetic runs in
the CUDA kernels; nothing here computes, and nothing falls back to the CPU: if
the compiled library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgva.so")

F32, BF16 = 0, 1
FLAG_FMA_PATH = 1
FLAG_TCGEN05_PATH = 2
DEVERR_RANGE, DEVERR_WAIT = 1, 2

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace too small",
           4: "CUDA error"}


class GVAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    """Mirror of gva_shape_t."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("G", ctypes.c_int32),
                ("d_h", ctypes.c_int32), ("d_n", ctypes.c_int32), ("d_r", ctypes.c_int32),
                ("cache_dtype", ctypes.c_int32), ("q_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("rope_base", ctypes.c_double), ("softmax_scale", ctypes.c_float),
                ("ctas_per_sm", ctypes.c_int32)]


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {dt}")


def make_shape(B, H, G, d_h, d_n, d_r, cache_dtype=torch.bfloat16, q_dtype=None,
               out_dtype=torch.float32, rope_base=10000.0, softmax_scale=0.0, flags=0,
               ctas_per_sm=0) -> Shape:
    q_dtype = cache_dtype if q_dtype is None else q_dtype
    return Shape(B, H, G, d_h, d_n, d_r, dtype_code(cache_dtype), dtype_code(q_dtype),
                 dtype_code(out_dtype), flags, float(rope_base), float(softmax_scale), ctas_per_sm)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgva.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """Open a build of the library and declare its C signatures."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m compressed_kv_cache_gva_b200._build`")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    L.gva_status_string.restype = ctypes.c_char_p
    L.gva_status_string.argtypes = [ctypes.c_int]
    L.gva_last_error.restype = ctypes.c_char_p
    L.gva_last_error.argtypes = []
    L.gva_absorb_query.restype = ctypes.c_int
    L.gva_absorb_query.argtypes = [SP, P, P, P, P, P]
    L.gva_append_cache.restype = ctypes.c_int
    L.gva_append_cache.argtypes = [SP, I32, P, P, P, P, I64, P, P, P, P]
    L.gva_decode_workspace_size.restype = SZ
    L.gva_decode_workspace_size.argtypes = [SP, I64]
    L.gva_decode_attention.restype = ctypes.c_int
    L.gva_decode_attention.argtypes = [SP, P, P, P, P, P, I64, I64, P, P, P, SZ, P]
    L.gqa_decode_attention.restype = ctypes.c_int
    L.gqa_decode_attention.argtypes = [SP, P, P, P, P, P, I64, I64, P, P, P, SZ, P]
    L.gva_decode_step.restype = ctypes.c_int
    L.gva_decode_step.argtypes = [SP, P, P, P, I32, P, P, P, P, P, P, I64, P, P, I64, P, P, P, P,
                                  P, SZ, P]
    L.gva_decode_workspace_size_multi.restype = SZ
    L.gva_decode_workspace_size_multi.argtypes = [SP, I32, I64]
    L.gva_decode_attention_multi.restype = ctypes.c_int
    L.gva_decode_attention_multi.argtypes = [SP, I32, P, P, P, P, P, I64, I64, P, P, P, SZ, P]
    L.gva_merge_states.restype = ctypes.c_int
    L.gva_merge_states.argtypes = [SP, I32, P, P, P, P, P]
    L.gva_shared_kv_decode_attention.restype = ctypes.c_int
    L.gva_shared_kv_decode_attention.argtypes = [SP, P, P, P, P, I64, I64, P, P, P, SZ, P]
    L.gqa_append_cache.restype = ctypes.c_int
    L.gqa_append_cache.argtypes = [SP, I32, P, P, P, P, I64, P, P, P, P]
    L.gqa_decode_step.restype = ctypes.c_int
    L.gqa_decode_step.argtypes = [SP, P, P, I32, P, P, P, P, P, P, I64, P, P, I64, P, P, P, P,
                                  P, SZ, P]
    L.gva_decode_attention_noalloc.restype = ctypes.c_int
    L.gva_decode_attention_noalloc.argtypes = [SP, P, P, P, P, P, I64, I64, P, P, P]
    L.gva_noalloc_status.restype = ctypes.c_int
    L.gva_noalloc_status.argtypes = [P, P]
    return L


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(st: int):
    if st != 0:
        raise GVAError(st, lib().gva_last_error().decode())


def absorb_query(shape: Shape, q, M, q_pos, q_abs, stream=None):
    _check(lib().gva_absorb_query(ctypes.byref(shape), _ptr(q), _ptr(M), _ptr(q_pos), _ptr(q_abs),
                                  _stream(stream)))


def append_cache(shape: Shape, v_new, kpe_new, slot, pos, V_cache, kr_cache, err_flag=None,
                 stream=None):
    N = slot.numel()
    _check(lib().gva_append_cache(ctypes.byref(shape), N, _ptr(v_new), _ptr(kpe_new), _ptr(slot),
                                  _ptr(pos), V_cache.shape[0], _ptr(V_cache), _ptr(kr_cache),
                                  _ptr(err_flag), _stream(stream)))


def decode_workspace_size(shape: Shape, max_total_tokens: int) -> int:
    return int(lib().gva_decode_workspace_size(ctypes.byref(shape), int(max_total_tokens)))


def new_workspace(shape: Shape, max_total_tokens: int, device=None) -> torch.Tensor:
    """A zeroed workspace (the status word must start at 0)."""
    n = decode_workspace_size(shape, max_total_tokens)
    if n == 0:
        raise GVAError(1, "invalid shape for a workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def workspace_status(ws: torch.Tensor) -> int:
    """Device status word of a workspace (synchronises)."""
    return int(ws[:4].view(torch.int32).item())


def decode_attention(shape: Shape, q_abs, V_cache, kr_cache, seq_offset, seq_len,
                     max_total_tokens: int, out, lse=None, workspace=None, stream=None):
    _check(lib().gva_decode_attention(
        ctypes.byref(shape), _ptr(q_abs), _ptr(V_cache), _ptr(kr_cache), _ptr(seq_offset),
        _ptr(seq_len), int(max_total_tokens), V_cache.shape[0], _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqa_decode_attention(shape: Shape, q, K_cache, V_cache, seq_offset, seq_len,
                         max_total_tokens: int, out, lse=None, workspace=None, stream=None):
    _check(lib().gqa_decode_attention(
        ctypes.byref(shape), _ptr(q), _ptr(K_cache), _ptr(V_cache), _ptr(seq_offset),
        _ptr(seq_len), int(max_total_tokens), V_cache.shape[0], _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqa_append_cache(shape: Shape, k_new, v_new, slot, pos, K_cache, V_cache, err_flag=None,
                     stream=None):
    """gqa_append_cache: the same-shape GQA baseline's append (key rotated over d_h)."""
    _check(lib().gqa_append_cache(ctypes.byref(shape), slot.numel(), _ptr(k_new), _ptr(v_new),
                                  _ptr(slot), _ptr(pos), V_cache.shape[0], _ptr(K_cache),
                                  _ptr(V_cache), _ptr(err_flag), _stream(stream)))


def gqa_decode_step(shape: Shape, q, q_pos, k_new, v_new, slot, pos, K_cache, V_cache,
                    seq_offset, seq_len, max_total_tokens: int, q_rot, out, lse=None,
                    err_flag=None, workspace=None, stream=None):
    """gqa_decode_step: rotate the queries, append the new tokens, GQA decode."""
    _check(lib().gqa_decode_step(
        ctypes.byref(shape), _ptr(q), _ptr(q_pos), slot.numel(), _ptr(k_new), _ptr(v_new),
        _ptr(slot), _ptr(pos), _ptr(K_cache), _ptr(V_cache), V_cache.shape[0], _ptr(seq_offset),
        _ptr(seq_len), int(max_total_tokens), _ptr(q_rot), _ptr(out), _ptr(lse), _ptr(err_flag),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_step(shape: Shape, q, M, q_pos, v_new, kpe_new, slot, pos, V_cache, kr_cache,
                seq_offset, seq_len, max_total_tokens: int, q_abs, out, lse=None, err_flag=None,
                workspace=None, stream=None):
    """gva_decode_step: append the new tokens, absorb the queries, decode."""
    _check(lib().gva_decode_step(
        ctypes.byref(shape), _ptr(q), _ptr(M), _ptr(q_pos), slot.numel(), _ptr(v_new),
        _ptr(kpe_new), _ptr(slot), _ptr(pos), _ptr(V_cache), _ptr(kr_cache), V_cache.shape[0],
        _ptr(seq_offset), _ptr(seq_len), int(max_total_tokens), _ptr(q_abs), _ptr(out), _ptr(lse),
        _ptr(err_flag), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def decode_workspace_size_multi(shape: Shape, n_query: int, max_total_tokens: int) -> int:
    return int(lib().gva_decode_workspace_size_multi(ctypes.byref(shape), int(n_query),
                                                     int(max_total_tokens)))


def decode_attention_multi(shape: Shape, n_query: int, q_abs, V_cache, kr_cache, seq_offset,
                           seq_len, max_total_tokens: int, out, lse=None, workspace=None,
                           stream=None):
    """gva_decode_attention_multi: n_query causal query tokens per sequence."""
    _check(lib().gva_decode_attention_multi(
        ctypes.byref(shape), int(n_query), _ptr(q_abs), _ptr(V_cache), _ptr(kr_cache),
        _ptr(seq_offset), _ptr(seq_len), int(max_total_tokens), V_cache.shape[0], _ptr(out),
        _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def shared_kv_decode_attention(shape: Shape, q, V_cache, seq_offset, seq_len,
                               max_total_tokens: int, out, lse=None, workspace=None, stream=None):
    """gva_shared_kv_decode_attention: keys are the values (M_h = I, d_r = 0)."""
    _check(lib().gva_shared_kv_decode_attention(
        ctypes.byref(shape), _ptr(q), _ptr(V_cache), _ptr(seq_offset), _ptr(seq_len),
        int(max_total_tokens), V_cache.shape[0], _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def merge_states(shape: Shape, outs, lses, out, lse=None, stream=None):
    """gva_merge_states: outs [R,B,H,d_h] float32, lses [R,B,H] float32."""
    _check(lib().gva_merge_states(ctypes.byref(shape), outs.shape[0], _ptr(outs), _ptr(lses),
                                  _ptr(out), _ptr(lse), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 << 20


def decode_attention_noalloc(shape: Shape, q_abs, V_cache, kr_cache, seq_offset, seq_len,
                             max_total_tokens: int, out, lse=None, stream=None):
    """gva_decode_attention_noalloc: the decode for callers that cannot allocate
    device memory; its scratch is a fixed array inside the library."""
    _check(lib().gva_decode_attention_noalloc(
        ctypes.byref(shape), _ptr(q_abs), _ptr(V_cache), _ptr(kr_cache), _ptr(seq_offset),
        _ptr(seq_len), int(max_total_tokens), V_cache.shape[0], _ptr(out), _ptr(lse),
        _stream(stream)))


def noalloc_status(stream=None) -> int:
    """Device status word of the last gva_decode_attention_noalloc call on the
    current device (enqueued behind it on the stream; synchronises to read it)."""
    buf = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib().gva_noalloc_status(_ptr(buf), _stream(stream)))
    return int(buf.item())


EXPORTS = ["gva_status_string", "gva_last_error", "gva_absorb_query", "gva_append_cache",
           "gva_decode_workspace_size", "gva_decode_attention", "gqa_decode_attention",
           "gva_decode_step", "gva_merge_states", "gva_decode_workspace_size_multi",
           "gva_decode_attention_multi", "gva_decode_attention_noalloc",
           "gva_shared_kv_decode_attention", "gqa_append_cache", "gqa_decode_step",
           "gva_noalloc_status"]
