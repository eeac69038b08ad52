"""Thin ctypes binding of librq (include/librq.h).

Argument marshalling only: every function forwards to the C entry point of
the same name in the in-tree ``librq.so``; tensors are passed as device
pointers and the stream defaults to torch's current CUDA stream.  Nothing
here computes any part of the method, and there is no fallback: if the
shared library is missing the import of this module's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

RQ_MAX_LOOPS = 32
RQ_BLOCK_TOKENS = 32
RQ_POLICY_LAST_LOOP = 0
RQ_POLICY_NEXT_LOOP = 1
RQ_POLICY_FIRST_LOOP = 2
RQ_POLICY_PREVIOUS_LOOP = 3
RQ_FLAG_UNIT_ALPHA = 1
RQ_FLAG_META16 = 2

RQ_OK = 0
RQ_ERR_INVALID_ARG = 1
RQ_ERR_UNSUPPORTED = 2
RQ_ERR_CAPACITY = 3
RQ_ERR_CUDA = 4
RQ_ERR_TIMEOUT = 5
RQ_ERR_WORKSPACE = 6

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "librq.so")

# Exported symbols of librq.h (tests check that the library exports them all).
SYMBOLS = (
    "rq_abi_version", "rq_status_string", "rq_layout_validate", "rq_cache_bytes",
    "rq_layer_bytes", "rq_cache_bind", "rq_quantize_anchor", "rq_quantize_append_residual",
    "rq_dequantize", "rq_decode_workspace_bytes", "rq_decode_workspace_init",
    "rq_decode_attention", "rq_decode_bf16_workspace_bytes", "rq_decode_attention_bf16",
    "rq_workspace_error", "rq_decode_splits", "rq_decode_attention_noalloc",
    "rq_quantize_append_loops", "rq_selftest_wait_timeout", "rq_cache_set_means",
    "rq_cache_set_rotations", "rq_plan_splits",
)


class rq_layout(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32), ("num_loops", ctypes.c_int32),
        ("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
        ("policy", ctypes.c_int32), ("flags", ctypes.c_int32),
        ("bits", ctypes.c_int32 * RQ_MAX_LOOPS), ("group", ctypes.c_int32 * RQ_MAX_LOOPS),
    ]


class rq_cache(ctypes.Structure):
    _fields_ = [
        ("layout", rq_layout), ("k_base", ctypes.c_void_p), ("v_base", ctypes.c_void_p),
        ("layer_bytes", ctypes.c_uint64), ("token_stride", ctypes.c_int64),
        ("comp_off", ctypes.c_uint64 * RQ_MAX_LOOPS),
        ("rec_bytes", ctypes.c_uint32 * RQ_MAX_LOOPS),
        ("k_means", ctypes.c_void_p), ("v_means", ctypes.c_void_p),
        ("k_rot", ctypes.c_void_p), ("v_rot", ctypes.c_void_p),
    ]


class RQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {rq_status_string(status)}")
        self.status = status


_lib: Optional[ctypes.CDLL] = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_U64 = ctypes.c_uint64
_F = ctypes.c_float


def load() -> ctypes.CDLL:
    """Loads the in-tree librq.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"librq.so not found at {LIB_PATH}; build it with "
                          "`python -m residual_bit_kv_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    LP = ctypes.POINTER(rq_layout)
    CP = ctypes.POINTER(rq_cache)
    sig = {
        "rq_abi_version": ([], _I32),
        "rq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "rq_layout_validate": ([LP], ctypes.c_int),
        "rq_cache_bytes": ([LP], _U64),
        "rq_layer_bytes": ([LP], _U64),
        "rq_cache_bind": ([LP, _P, _P, CP], ctypes.c_int),
        "rq_cache_set_means": ([CP, _P, _P], ctypes.c_int),
        "rq_cache_set_rotations": ([CP, _P, _P], ctypes.c_int),
        "rq_plan_splits": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                            ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)],
                           ctypes.c_int),
        "rq_quantize_anchor": ([CP, _I32, _I32, _P, _I32, _I32, _P], ctypes.c_int),
        "rq_quantize_append_residual": ([CP, _I32, _I32, _I32, _P, _I32, _I32, _P], ctypes.c_int),
        "rq_quantize_append_loops": ([CP, _I32, _P, _P, _I32, _I32, _P], ctypes.c_int),
        "rq_dequantize": ([CP, _I32, _I32, _I32, _I32, _I32, _P, _P], ctypes.c_int),
        "rq_decode_workspace_bytes": ([LP, _I32], _U64),
        "rq_decode_workspace_init": ([_P, _U64, _P], ctypes.c_int),
        "rq_decode_attention": ([CP, _I32, _I32, _P, _P, _I32, _P, _P, _F, _P, _P, _U64, _P],
                                ctypes.c_int),
        "rq_decode_bf16_workspace_bytes": ([_I32, _I32, _I32, _I32], _U64),
        "rq_decode_attention_bf16": ([_I32, _I32, _I32, _P, _P, _P, _I64, _P, _I32, _P, _P, _F,
                                      _P, _P, _U64, _P], ctypes.c_int),
        "rq_workspace_error": ([_P, _U64, _P], ctypes.c_int),
        "rq_selftest_wait_timeout": ([_P, ctypes.c_uint64, ctypes.c_int32, _P], ctypes.c_int),
        "rq_decode_splits": ([LP, _I32], _I32),
        "rq_decode_attention_noalloc": ([CP, _I32, _I32, _P, _P, _I32, _P, _P, _F, _P, _P],
                                        ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


# ------------------------------------------------------------------ helpers --

def _ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> None:
    if status != RQ_OK:
        raise RQError(status, what)


def make_layout(num_layers: int, num_loops: int, batch: int, kv_heads: int, head_dim: int,
                max_tokens: int, bits: Sequence[int], group: Sequence[int],
                policy: int = RQ_POLICY_LAST_LOOP, flags: int = 0) -> rq_layout:
    lay = rq_layout()
    lay.num_layers, lay.num_loops, lay.batch, lay.kv_heads = num_layers, num_loops, batch, kv_heads
    lay.head_dim, lay.max_tokens, lay.policy, lay.flags = head_dim, max_tokens, policy, flags
    for r in range(min(num_loops, RQ_MAX_LOOPS, len(bits), len(group))):
        lay.bits[r] = int(bits[r])
        lay.group[r] = int(group[r])
    return lay


# --------------------------------------------------------------- entry points --

def rq_abi_version() -> int:
    return int(load().rq_abi_version())


def rq_status_string(status: int) -> str:
    return load().rq_status_string(int(status)).decode()


def rq_layout_validate(layout: rq_layout) -> int:
    return int(load().rq_layout_validate(ctypes.byref(layout)))


def rq_cache_bytes(layout: rq_layout) -> int:
    return int(load().rq_cache_bytes(ctypes.byref(layout)))


def rq_layer_bytes(layout: rq_layout) -> int:
    return int(load().rq_layer_bytes(ctypes.byref(layout)))


def rq_cache_bind(layout: rq_layout, k_base, v_base) -> rq_cache:
    c = rq_cache()
    _check(load().rq_cache_bind(ctypes.byref(layout), _ptr(k_base), _ptr(v_base), ctypes.byref(c)),
           "rq_cache_bind")
    return c


def rq_cache_set_means(cache: rq_cache, k_means, v_means) -> None:
    """k_means, v_means: fp32 [num_layers, num_loops, kv_heads, head_dim] device
    tensors (rotated domain) or None."""
    _check(load().rq_cache_set_means(ctypes.byref(cache),
                                     None if k_means is None else _ptr(k_means),
                                     None if v_means is None else _ptr(v_means)),
           "rq_cache_set_means")


def rq_cache_set_rotations(cache: rq_cache, k_rot, v_rot) -> None:
    """k_rot, v_rot: binary16 (torch.float16 or 16-bit words) device tensors
    [num_layers, kv_heads, head_dim, head_dim], row i of a matrix giving
    output channel i, or None for the Hadamard transform of that side."""
    _check(load().rq_cache_set_rotations(ctypes.byref(cache),
                                         None if k_rot is None else _ptr(k_rot),
                                         None if v_rot is None else _ptr(v_rot)),
           "rq_cache_set_rotations")


def rq_quantize_anchor(cache: rq_cache, layer: int, kv: int, x, t0: int, n: int,
                       stream=None) -> None:
    _check(load().rq_quantize_anchor(ctypes.byref(cache), layer, kv, _ptr(x), t0, n,
                                     _stream(stream)), "rq_quantize_anchor")


def rq_quantize_append_residual(cache: rq_cache, layer: int, kv: int, loop: int, x, t0: int,
                                n: int, stream=None) -> None:
    _check(load().rq_quantize_append_residual(ctypes.byref(cache), layer, kv, loop, _ptr(x), t0,
                                              n, _stream(stream)), "rq_quantize_append_residual")


def rq_quantize_append_loops(cache: rq_cache, layer: int, xk, xv, t0: int, n: int,
                             stream=None) -> None:
    """xk, xv: bf16 [num_loops, batch, kv_heads, n, head_dim] device tensors (or None)."""
    _check(load().rq_quantize_append_loops(ctypes.byref(cache), layer,
                                           None if xk is None else _ptr(xk),
                                           None if xv is None else _ptr(xv), t0, n,
                                           _stream(stream)), "rq_quantize_append_loops")


def rq_dequantize(cache: rq_cache, layer: int, kv: int, loop: int, t0: int, n: int, out,
                  stream=None) -> None:
    _check(load().rq_dequantize(ctypes.byref(cache), layer, kv, loop, t0, n, _ptr(out),
                                _stream(stream)), "rq_dequantize")


def rq_decode_workspace_bytes(layout: rq_layout, max_seq_len: int) -> int:
    return int(load().rq_decode_workspace_bytes(ctypes.byref(layout), max_seq_len))


def rq_decode_workspace_init(workspace, ws_bytes: int, stream=None) -> None:
    _check(load().rq_decode_workspace_init(_ptr(workspace), ws_bytes, _stream(stream)),
           "rq_decode_workspace_init")


def rq_decode_attention(cache: rq_cache, layer: int, loop: int, q, seq_lens, max_seq_len: int,
                        k_cur, v_cur, softmax_scale: float, out, workspace, ws_bytes: int,
                        stream=None) -> None:
    _check(load().rq_decode_attention(ctypes.byref(cache), layer, loop, _ptr(q), _ptr(seq_lens),
                                      max_seq_len, _ptr(k_cur), _ptr(v_cur), softmax_scale,
                                      _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "rq_decode_attention")


def rq_decode_bf16_workspace_bytes(batch: int, heads: int, head_dim: int, max_seq_len: int) -> int:
    return int(load().rq_decode_bf16_workspace_bytes(batch, heads, head_dim, max_seq_len))


def rq_decode_attention_bf16(batch: int, heads: int, head_dim: int, q, k, v, token_stride: int,
                             seq_lens, max_seq_len: int, k_cur, v_cur, softmax_scale: float, out,
                             workspace, ws_bytes: int, stream=None) -> None:
    _check(load().rq_decode_attention_bf16(batch, heads, head_dim, _ptr(q), _ptr(k), _ptr(v),
                                           token_stride, _ptr(seq_lens), max_seq_len, _ptr(k_cur),
                                           _ptr(v_cur), softmax_scale, _ptr(out), _ptr(workspace),
                                           ws_bytes, _stream(stream)), "rq_decode_attention_bf16")


def rq_plan_splits(rows: int, max_seq_len: int, ctas_per_sm: int, sms: int):
    """(splits, chunks_per_split) of the decode split plan for a device with
    `sms` multiprocessors (host logic only)."""
    s = ctypes.c_int32()
    c = ctypes.c_int32()
    _check(load().rq_plan_splits(rows, max_seq_len, ctas_per_sm, sms, ctypes.byref(s),
                                 ctypes.byref(c)), "rq_plan_splits")
    return s.value, c.value


def rq_workspace_error(workspace, ws_bytes: int, stream=None) -> int:
    return int(load().rq_workspace_error(_ptr(workspace), ws_bytes, _stream(stream)))


def rq_selftest_wait_timeout(workspace, ws_bytes: int, limit_ms: int, stream=None) -> None:
    _check(load().rq_selftest_wait_timeout(_ptr(workspace), ws_bytes, limit_ms, _stream(stream)),
           "rq_selftest_wait_timeout")


def rq_decode_splits(layout: rq_layout, max_seq_len: int) -> int:
    return int(load().rq_decode_splits(ctypes.byref(layout), max_seq_len))


def rq_decode_attention_noalloc(cache: rq_cache, layer: int, loop: int, q, seq_lens,
                                max_seq_len: int, k_cur, v_cur, softmax_scale: float, out,
                                stream=None) -> None:
    """rq_decode_attention without a workspace, for callers that cannot
    allocate device memory; see include/librq.h."""
    _check(load().rq_decode_attention_noalloc(ctypes.byref(cache), layer, loop, _ptr(q),
                                              _ptr(seq_lens), max_seq_len, _ptr(k_cur),
                                              _ptr(v_cur), softmax_scale, _ptr(out),
                                              _stream(stream)), "rq_decode_attention_noalloc")
