"""ctypes binding of libdz (include/dz.h), argument marshalling only.

Every function has the name and argument order of its C counterpart.  Tensor
arguments may be torch tensors (their ``data_ptr()`` is passed) or raw device
addresses (int).  A non-OK status raises ``DzError``.  The library is loaded
from this package directory; if it is missing the import fails loudly -- there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdz.so")

DZ_OK = 0
DZ_ERR_INVALID_ARG = 1
DZ_ERR_ALIGNMENT = 2
DZ_ERR_SHAPE = 3
DZ_ERR_CAPACITY = 4
DZ_ERR_CUDA = 5
DZ_ERR_UNSUPPORTED = 6
DZ_ERR_TIMEOUT = 7
DZ_ERR_BOUNDS = 8

DZ_MODE_DECODE = 0
DZ_MODE_TEACHER_FORCING = 1
DZ_MODE_PREFILL = 2
DZ_MODE_CROSS = 3
DZ_MODE_ROTATED = 0x100  # flag: q and the call's own k are already rotated

# Every entry point include/dz.h declares.
EXPORTS = [
    "dz_attn_create", "dz_attn_destroy", "dz_rope3d", "dz_chunk_attn_forward",
    "dz_kvcache_append", "dz_kvcache_replace", "dz_attn_sync_status", "dz_status_string",
    "dz_chunk_attn_forward_noalloc", "dz_qkv_rope", "dz_chunk_attn_forward_lse",
    "dz_chunk_attn_backward", "dz_chunk_attn_forward_e4m3", "dz_quantize_e4m3",
    "dz_rope3d_e4m3",
]


class DzError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class dz_attn_desc(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("rope_pairs_t", ctypes.c_int32), ("rope_pairs_h", ctypes.c_int32),
        ("rope_pairs_w", ctypes.c_int32),
        ("max_batch", ctypes.c_int32), ("max_q_tokens", ctypes.c_int32),
        ("max_pos_t", ctypes.c_int32), ("max_pos_h", ctypes.c_int32),
        ("max_pos_w", ctypes.c_int32), ("prerotate_tokens", ctypes.c_int32),
    ]


class dz_chunk_layout(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32), ("batch", ctypes.c_int32),
        ("frames_per_chunk", ctypes.c_int32), ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32), ("n_action", ctypes.c_int32),
        ("num_chunks", ctypes.c_int32), ("t_offset", ctypes.c_int32),
        ("kv_len", ctypes.c_int32),
    ]


class dz_kvcache(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("capacity_tokens", ctypes.c_int32),
        ("len_tokens", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
    ]


_lib: Optional[ctypes.CDLL] = None


def bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the argument and result types of every entry point on a loaded libdz."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.dz_attn_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(dz_attn_desc)]
    lib.dz_attn_destroy.argtypes = [vp]
    lib.dz_rope3d.argtypes = [vp, vp, vp, i32, i32, ctypes.POINTER(dz_chunk_layout), i32, vp]
    lib.dz_chunk_attn_forward.argtypes = [vp, vp, vp, vp, ctypes.POINTER(dz_kvcache),
                                          ctypes.POINTER(dz_chunk_layout), vp, vp]
    lib.dz_chunk_attn_forward_noalloc.argtypes = [
        ctypes.POINTER(dz_attn_desc), vp, vp, vp, ctypes.POINTER(dz_kvcache),
        ctypes.POINTER(dz_chunk_layout), vp, vp]
    lib.dz_kvcache_append.argtypes = [vp, ctypes.POINTER(dz_kvcache), vp, vp, vp]
    lib.dz_kvcache_replace.argtypes = [vp, ctypes.POINTER(dz_kvcache), i32, vp, vp, vp]
    lib.dz_qkv_rope.argtypes = [vp, vp, vp, i32, i32, i32, ctypes.POINTER(dz_chunk_layout), i32,
                                vp, vp, vp, ctypes.POINTER(dz_kvcache), vp]
    lib.dz_chunk_attn_forward_lse.argtypes = [vp, vp, vp, vp, ctypes.POINTER(dz_chunk_layout),
                                              vp, vp, vp]
    lib.dz_chunk_attn_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp,
                                           ctypes.POINTER(dz_chunk_layout), vp, vp, vp, vp]
    lib.dz_chunk_attn_forward_e4m3.argtypes = [vp, vp, vp, vp, ctypes.POINTER(dz_kvcache),
                                               ctypes.POINTER(dz_chunk_layout), ctypes.c_float,
                                               ctypes.c_float, vp, vp]
    lib.dz_quantize_e4m3.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.c_float, vp]
    lib.dz_rope3d_e4m3.argtypes = [vp, vp, vp, i32, i32, ctypes.POINTER(dz_chunk_layout), i32,
                                   ctypes.c_float, vp]
    lib.dz_attn_sync_status.argtypes = [vp, vp]
    lib.dz_status_string.argtypes = [ctypes.c_int]
    lib.dz_status_string.restype = ctypes.c_char_p
    for name in EXPORTS:
        if name != "dz_status_string":
            getattr(lib, name).restype = ctypes.c_int
    return lib


def load() -> ctypes.CDLL:
    """Load libdz.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdz.so is not built ({LIB_PATH}); run "
                          "python -m causal_video_diffusion_rope_b200.build")
    _lib = bind(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(status: int) -> str:
    return load().dz_status_string(int(status)).decode()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) if torch.cuda.is_available() else None
    if hasattr(s, "cuda_stream"):
        return int(s.cuda_stream)
    return int(s)


def _check(st: int, where: str) -> None:
    if st != DZ_OK:
        raise DzError(st, where)


def make_desc(num_heads: int = 40, max_batch: int = 2, max_q_tokens: int = 8192,
              max_pos_t: int = 4096, max_pos_h: int = 256, max_pos_w: int = 256,
              rope_base: float = 10000.0, pairs=(22, 21, 21),
              prerotate_tokens: int = 0) -> dz_attn_desc:
    return dz_attn_desc(num_heads, 128, rope_base, pairs[0], pairs[1], pairs[2], max_batch,
                        max_q_tokens, max_pos_t, max_pos_h, max_pos_w, prerotate_tokens)


def make_layout(mode: int, batch: int, frames_per_chunk: int, grid_h: int, grid_w: int,
                n_action: int, num_chunks: int, t_offset: int = 0, kv_len: int = 0
                ) -> dz_chunk_layout:
    return dz_chunk_layout(mode, batch, frames_per_chunk, grid_h, grid_w, n_action, num_chunks,
                           t_offset, kv_len)


def layout_from(lay) -> dz_chunk_layout:
    """dz_chunk_layout from an object with the same field names (e.g. synth.Layout)."""
    return make_layout(lay.mode, lay.batch, lay.frames_per_chunk, lay.grid_h, lay.grid_w,
                       lay.n_action, lay.num_chunks, lay.t_offset, lay.kv_len)


def make_cache(k, v, batch: int, capacity_tokens: int, len_tokens: int, chunk_len: int
               ) -> dz_kvcache:
    return dz_kvcache(_ptr(k), _ptr(v), batch, capacity_tokens, len_tokens, chunk_len)


# ---------------------------------------------------------------- entry points

def dz_attn_create(desc: dz_attn_desc) -> int:
    h = ctypes.c_void_p()
    _check(load().dz_attn_create(ctypes.byref(h), ctypes.byref(desc)), "dz_attn_create")
    return h.value


def dz_attn_destroy(handle: int) -> None:
    _check(load().dz_attn_destroy(handle), "dz_attn_destroy")


def dz_rope3d(handle: int, x, y, B: int, S: int, layout: dz_chunk_layout, first_chunk: int,
              stream=None) -> None:
    _check(load().dz_rope3d(handle, _ptr(x), _ptr(y), B, S, ctypes.byref(layout), first_chunk,
                            _stream(stream)), "dz_rope3d")


def dz_chunk_attn_forward(handle: int, q, k, v, cache: Optional[dz_kvcache],
                          layout: dz_chunk_layout, out, stream=None) -> None:
    cptr = ctypes.byref(cache) if cache is not None else None
    _check(load().dz_chunk_attn_forward(handle, _ptr(q), _ptr(k), _ptr(v), cptr,
                                        ctypes.byref(layout), _ptr(out), _stream(stream)),
           "dz_chunk_attn_forward")


def dz_chunk_attn_forward_e4m3(handle: int, q8, k8, v, cache: Optional[dz_kvcache],
                               layout: dz_chunk_layout, q_scale: float, k_scale: float, out,
                               stream=None) -> None:
    cptr = ctypes.byref(cache) if cache is not None else None
    _check(load().dz_chunk_attn_forward_e4m3(handle, _ptr(q8), _ptr(k8), _ptr(v), cptr,
                                             ctypes.byref(layout), q_scale, k_scale, _ptr(out),
                                             _stream(stream)),
           "dz_chunk_attn_forward_e4m3")


def dz_rope3d_e4m3(handle: int, x, y8, B: int, S: int, layout: dz_chunk_layout, first_chunk: int,
                   scale: float, stream=None) -> None:
    _check(load().dz_rope3d_e4m3(handle, _ptr(x), _ptr(y8), B, S, ctypes.byref(layout), first_chunk,
                                 scale, _stream(stream)), "dz_rope3d_e4m3")


def dz_quantize_e4m3(handle: int, x, y, n: int, scale: float, stream=None) -> None:
    _check(load().dz_quantize_e4m3(handle, _ptr(x), _ptr(y), n, scale, _stream(stream)),
           "dz_quantize_e4m3")


def dz_chunk_attn_forward_noalloc(desc: dz_attn_desc, q, k, v, cache: Optional[dz_kvcache],
                                  layout: dz_chunk_layout, out, stream=None) -> None:
    """Attention for callers that cannot allocate device memory (no handle; static scratch)."""
    cptr = ctypes.byref(cache) if cache is not None else None
    _check(load().dz_chunk_attn_forward_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                                cptr, ctypes.byref(layout), _ptr(out),
                                                _stream(stream)),
           "dz_chunk_attn_forward_noalloc")


def dz_kvcache_append(handle: int, cache: dz_kvcache, k, v, stream=None) -> None:
    _check(load().dz_kvcache_append(handle, ctypes.byref(cache), _ptr(k), _ptr(v),
                                    _stream(stream)), "dz_kvcache_append")


def dz_kvcache_replace(handle: int, cache: dz_kvcache, chunk_index: int, k, v,
                       stream=None) -> None:
    _check(load().dz_kvcache_replace(handle, ctypes.byref(cache), chunk_index, _ptr(k), _ptr(v),
                                     _stream(stream)), "dz_kvcache_replace")


def dz_qkv_rope(handle: int, x, w, B: int, S: int, d_model: int, layout: dz_chunk_layout,
                first_chunk: int, q_out, k_out, v_out, cache: Optional[dz_kvcache] = None,
                stream=None) -> None:
    """QKV projection with the rotation (and optionally the cache append) fused in."""
    cptr = ctypes.byref(cache) if cache is not None else None
    _check(load().dz_qkv_rope(handle, _ptr(x), _ptr(w), B, S, d_model, ctypes.byref(layout),
                              first_chunk, _ptr(q_out), _ptr(k_out), _ptr(v_out), cptr,
                              _stream(stream)), "dz_qkv_rope")


def dz_chunk_attn_forward_lse(handle: int, q, k, v, layout: dz_chunk_layout, out, lse,
                              stream=None) -> None:
    """Training-form forward: also writes each query row's log2 softmax normaliser."""
    _check(load().dz_chunk_attn_forward_lse(handle, _ptr(q), _ptr(k), _ptr(v),
                                            ctypes.byref(layout), _ptr(out), _ptr(lse),
                                            _stream(stream)), "dz_chunk_attn_forward_lse")


def dz_chunk_attn_backward(handle: int, q, k, v, out, dout, lse, layout: dz_chunk_layout,
                           dq, dk, dv, stream=None) -> None:
    """Gradients of sum(dout * out) with respect to the unrotated q, k and v."""
    _check(load().dz_chunk_attn_backward(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                         _ptr(lse), ctypes.byref(layout), _ptr(dq), _ptr(dk),
                                         _ptr(dv), _stream(stream)), "dz_chunk_attn_backward")


def dz_attn_sync_status(handle: int, stream=None) -> None:
    _check(load().dz_attn_sync_status(handle, _stream(stream)), "dz_attn_sync_status")


def dz_status_string(status: int) -> str:
    return status_string(status)
