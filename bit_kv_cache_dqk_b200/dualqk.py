"""Thin ctypes binding of libdualqk (include/dualqk.h): same names, argument
marshalling only.  Every step of the decode path runs in the library's CUDA
kernels; there is no Python or CPU fallback -- if libdualqk.so is missing the
import fails.

Tensors may be passed as torch tensors (their ``data_ptr()`` is taken) or as
raw integer addresses.  ``stream`` defaults to torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdualqk.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libdualqk.so not built at {_LIB_PATH}; run bit_kv_cache_dqk_b200.build.build()")

_lib = C.CDLL(_LIB_PATH)

DQK_OK, DQK_ERR_INVALID_ARG, DQK_ERR_UNSUPPORTED, DQK_ERR_WORKSPACE_TOO_SMALL = 0, 1, 2, 3
DQK_ERR_CUDA, DQK_ERR_DEVICE_BOUNDS, DQK_ERR_TIMEOUT = 4, 5, 6
DQK_F32, DQK_BF16 = 0, 1

EXPORTED = ["dqk_block_bytes", "dqk_append", "dqk_decode_workspace_size", "dqk_decode",
            "dqk_decode_step", "dqk_decode_partial", "dqk_merge_partials", "dqk_test_decode_stall",
            "dqk_decode_noalloc", "dqk_bf16_block_bytes", "dqk_bf16_append",
            "dqk_bf16_decode_workspace_size", "dqk_bf16_decode", "dqk_last_device_error", "dqk_status_string"]

DQK_NOALLOC_WORKSPACE_BYTES = 8 << 20


class dqk_layer_desc(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("num_q_heads", C.c_int), ("num_kv_heads", C.c_int),
                ("page_size", C.c_int), ("group_size", C.c_int), ("v_ch0_protect", C.c_int),
                ("t_k", C.c_void_p), ("t_q", C.c_void_p), ("pool", C.c_void_p),
                ("num_pages", C.c_longlong)]


_P = C.c_void_p
_D = C.POINTER(dqk_layer_desc)
_lib.dqk_block_bytes.restype = C.c_size_t
_lib.dqk_block_bytes.argtypes = [_D]
_lib.dqk_append.restype = C.c_int
_lib.dqk_append.argtypes = [_D, _P, _P, C.c_int, C.c_int, _P, _P, C.c_int, _P, C.c_int, _P]
_lib.dqk_decode_workspace_size.restype = C.c_size_t
_lib.dqk_decode_workspace_size.argtypes = [_D, C.c_int, C.c_int]
for _n in ("dqk_decode", "dqk_decode_partial", "dqk_test_decode_stall"):
    getattr(_lib, _n).restype = C.c_int
    getattr(_lib, _n).argtypes = [_D, _P, C.c_int, C.c_int, _P, _P, C.c_int, C.c_int, _P, _P, _P,
                                  C.c_size_t, _P]
_lib.dqk_merge_partials.restype = C.c_int
_lib.dqk_merge_partials.argtypes = [_P, C.c_int, C.c_int, C.c_int, C.c_int, _P, _P]
_lib.dqk_decode_step.restype = C.c_int
_lib.dqk_decode_step.argtypes = [_D, _P, _P, C.c_int, _P, _P, C.c_int, _P, C.c_int, C.c_int, _P, _P, C.c_int,
                                 C.c_int, _P, _P, _P, C.c_size_t, _P]
_lib.dqk_decode_noalloc.restype = C.c_int
_lib.dqk_decode_noalloc.argtypes = [_D, _P, C.c_int, C.c_int, _P, _P, C.c_int, C.c_int, _P, _P, _P]
_lib.dqk_bf16_block_bytes.restype = C.c_size_t
_lib.dqk_bf16_block_bytes.argtypes = [_D]
_lib.dqk_bf16_append.restype = C.c_int
_lib.dqk_bf16_append.argtypes = [_D, _P, _P, C.c_int, C.c_int, _P, _P, C.c_int, _P, C.c_int, _P]
_lib.dqk_bf16_decode_workspace_size.restype = C.c_size_t
_lib.dqk_bf16_decode_workspace_size.argtypes = [_D, C.c_int, C.c_int]
_lib.dqk_bf16_decode.restype = C.c_int
_lib.dqk_bf16_decode.argtypes = [_D, _P, C.c_int, C.c_int, _P, _P, C.c_int, _P, _P, C.c_size_t, _P]
_lib.dqk_last_device_error.restype = C.c_int
_lib.dqk_last_device_error.argtypes = [_P]
_lib.dqk_status_string.restype = C.c_char_p
_lib.dqk_status_string.argtypes = [C.c_int]


class DQKError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {dqk_status_string(status)}")
        self.status = status


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str, raise_on_error: bool):
    if raise_on_error and status != DQK_OK:
        raise DQKError(status, where)
    return status


def layer_desc(head_dim, num_q_heads, num_kv_heads, t_k, t_q, pool, num_pages, v_ch0_protect=0,
               page_size=16, group_size=32) -> dqk_layer_desc:
    return dqk_layer_desc(head_dim, num_q_heads, num_kv_heads, page_size, group_size, v_ch0_protect,
                          _addr(t_k), _addr(t_q), _addr(pool), num_pages)


def dqk_block_bytes(layer: dqk_layer_desc) -> int:
    return int(_lib.dqk_block_bytes(C.byref(layer)))


def dqk_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages,
               stream=None, raise_on_error=True) -> int:
    st = _lib.dqk_append(C.byref(layer), _addr(k), _addr(v), dtype, batch, _addr(new_lens),
                         _addr(seq_lens_before), max_new, _addr(page_table), max_pages, _stream(stream))
    return _check(st, "dqk_append", raise_on_error)


def dqk_decode_workspace_size(layer, batch, max_pages) -> int:
    return int(_lib.dqk_decode_workspace_size(C.byref(layer), batch, max_pages))


def _decode(fn, name, layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out,
            sel_out, workspace, workspace_bytes, stream, raise_on_error):
    st = fn(C.byref(layer), _addr(q), q_dtype, batch, _addr(seq_lens), _addr(page_table), max_pages,
            sparsity_pct, _addr(out), _addr(sel_out), _addr(workspace), workspace_bytes, _stream(stream))
    return _check(st, name, raise_on_error)


def dqk_decode(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out, sel_out,
               workspace, workspace_bytes, stream=None, raise_on_error=True) -> int:
    return _decode(_lib.dqk_decode, "dqk_decode", layer, q, q_dtype, batch, seq_lens, page_table,
                   max_pages, sparsity_pct, out, sel_out, workspace, workspace_bytes, stream, raise_on_error)


def dqk_decode_step(layer, k, v, kv_dtype, new_lens, seq_lens_before, max_new, q, q_dtype, batch, seq_lens,
                    page_table, max_pages, sparsity_pct, out, sel_out, workspace, workspace_bytes, stream=None,
                    raise_on_error=True) -> int:
    st = _lib.dqk_decode_step(C.byref(layer), _addr(k), _addr(v), kv_dtype, _addr(new_lens),
                              _addr(seq_lens_before), max_new, _addr(q), q_dtype, batch, _addr(seq_lens),
                              _addr(page_table), max_pages, sparsity_pct, _addr(out), _addr(sel_out),
                              _addr(workspace), workspace_bytes, _stream(stream))
    return _check(st, "dqk_decode_step", raise_on_error)


def dqk_decode_partial(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, part, sel_out,
                       workspace, workspace_bytes, stream=None, raise_on_error=True) -> int:
    return _decode(_lib.dqk_decode_partial, "dqk_decode_partial", layer, q, q_dtype, batch, seq_lens, page_table,
                   max_pages, sparsity_pct, part, sel_out, workspace, workspace_bytes, stream, raise_on_error)


def dqk_merge_partials(parts, n_parts, batch, num_q_heads, head_dim, out, stream=None, raise_on_error=True) -> int:
    st = _lib.dqk_merge_partials(_addr(parts), n_parts, batch, num_q_heads, head_dim, _addr(out), _stream(stream))
    return _check(st, "dqk_merge_partials", raise_on_error)


def dqk_test_decode_stall(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out,
                          sel_out, workspace, workspace_bytes, stream=None, raise_on_error=True) -> int:
    """Test only: dqk_decode with a stalled ring stage and 1 ms ring waits
    (see include/dualqk.h); the device error word then reads DQK_ERR_TIMEOUT."""
    return _decode(_lib.dqk_test_decode_stall, "dqk_test_decode_stall", layer, q, q_dtype, batch, seq_lens,
                   page_table, max_pages, sparsity_pct, out, sel_out, workspace, workspace_bytes, stream,
                   raise_on_error)


def dqk_decode_noalloc(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out,
                       sel_out, stream=None, raise_on_error=True) -> int:
    """dqk_decode for callers that cannot provide a workspace (the library's
    static scratch is used; see include/dualqk.h)."""
    st = _lib.dqk_decode_noalloc(C.byref(layer), _addr(q), q_dtype, batch, _addr(seq_lens), _addr(page_table),
                                 max_pages, sparsity_pct, _addr(out), _addr(sel_out), _stream(stream))
    return _check(st, "dqk_decode_noalloc", raise_on_error)


def dqk_bf16_block_bytes(layer: dqk_layer_desc) -> int:
    return int(_lib.dqk_bf16_block_bytes(C.byref(layer)))


def dqk_bf16_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages,
                    stream=None, raise_on_error=True) -> int:
    st = _lib.dqk_bf16_append(C.byref(layer), _addr(k), _addr(v), dtype, batch, _addr(new_lens),
                              _addr(seq_lens_before), max_new, _addr(page_table), max_pages, _stream(stream))
    return _check(st, "dqk_bf16_append", raise_on_error)


def dqk_bf16_decode_workspace_size(layer, batch, max_pages) -> int:
    return int(_lib.dqk_bf16_decode_workspace_size(C.byref(layer), batch, max_pages))


def dqk_bf16_decode(layer, q, q_dtype, batch, seq_lens, page_table, max_pages, out, workspace, workspace_bytes,
                    stream=None, raise_on_error=True) -> int:
    st = _lib.dqk_bf16_decode(C.byref(layer), _addr(q), q_dtype, batch, _addr(seq_lens), _addr(page_table),
                              max_pages, _addr(out), _addr(workspace), workspace_bytes, _stream(stream))
    return _check(st, "dqk_bf16_decode", raise_on_error)


def dqk_last_device_error(stream=None) -> int:
    return int(_lib.dqk_last_device_error(_stream(stream)))


def dqk_status_string(status: int) -> str:
    return _lib.dqk_status_string(status).decode()


def library_path() -> str:
    return _LIB_PATH
