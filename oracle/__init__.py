"""CPU oracle for the ResidualQuant KV-cache hot path.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product library (``librq``) never imports, links or executes
anything here, and this package imports nothing from the product.

The arithmetic lives in plain C (``rqo.c``, single-threaded, built with
``-ffp-contract=off``); this module only marshals numpy arrays.  Citations
``[RQ §x]`` refer to "ResidualQuant: KV Cache Quantization for Looped
Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).

Array conventions (all C-contiguous):
  x      uint16 bf16 bits, [L, N, D]: loop l, row n (rows are (b, h, t) in
         that nesting order), channel d.  Loop L-1 is the final-loop anchor.
  codes  uint32 [N, D*bits/32]; meta uint32 [N, D/group] (fp16 scale in the
         low half, fp16 offset in the high half); alpha uint16 [N] (bf16).
  quantize_m8: the 16-bit-metadata variant, meta uint16 [D/group] (scale
         byte, offset byte); see rqo.h.

Parity unpinned: nothing here is pinned against learned rotations, real
model KV, or the pages' accuracy / NMSE / throughput numbers; the pins are
closed forms, invariants, brute force and the pages' storage accounting.
"""
from __future__ import annotations

import ctypes
import functools
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rqo.c")
_LIB_PATH = os.path.join(_HERE, "librqo.so")

POLICY_LAST = "last"           # shared anchor at the final loop [RQ §3.2 Last-loop]
POLICY_NEXT = "next"           # chain toward the final loop [RQ §5.2 Next-loop]
POLICY_FIRST = "first"         # shared anchor at the first loop [RQ §3.2 First-loop]
POLICY_PREVIOUS = "previous"   # chain toward the first loop [RQ §3.1, §3.2 Previous-loop]
POLICIES = (POLICY_LAST, POLICY_NEXT, POLICY_FIRST, POLICY_PREVIOUS)


def anchor_loop(L: int, policy: str) -> int:
    """Index of the anchor loop: the final loop for Last-/Next-loop, the first
    for First-/Previous-loop [RQ §3.2, App. D]."""
    return L - 1 if policy in (POLICY_LAST, POLICY_NEXT) else 0


def is_chained(policy: str) -> bool:
    return policy in (POLICY_NEXT, POLICY_PREVIOUS)


def reference_loop(L: int, r: int, policy: str) -> int:
    """The loop whose reconstruction loop r references [RQ §3.2, App. D]:
    the anchor (shared policies), r + 1 (Next-loop) or r - 1 (Previous-loop)."""
    if policy == POLICY_NEXT:
        return r + 1
    if policy == POLICY_PREVIOUS:
        return r - 1
    return anchor_loop(L, policy)


def encode_order(L: int, policy: str) -> List[int]:
    """Residual loops in an order where every reference is encoded first:
    away from the anchor."""
    a = anchor_loop(L, policy)
    return list(range(a - 1, -1, -1)) if a == L - 1 else list(range(1, L))

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile rqo.c into librqo.so next to it (gcc, no fused multiply-add)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                                  os.path.getmtime(os.path.join(_HERE, "rqo.h"))))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib: Optional[ctypes.CDLL] = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_D = ctypes.c_double


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        h = ctypes.CDLL(build())
        sig = {
            "rqo_bf16_to_f32": ([ctypes.c_uint16], _F),
            "rqo_f32_to_bf16": ([_F], ctypes.c_uint16),
            "rqo_f16_to_f32": ([ctypes.c_uint16], _F),
            "rqo_f32_to_f16": ([_F], ctypes.c_uint16),
            "rqo_rot_scale": ([_I], _F),
            "rqo_fwht_f32": ([_P, _I], None),
            "rqo_fwht_f64": ([_P, _I], None),
            "rqo_fwht_rows_f64": ([_P, _I64, _I], None),
            "rqo_dot_f32": ([_P, _P, _I], _F),
            "rqo_quantize": ([_P, _I, _I, _I, _P, _P, _P], None),
            "rqo_encode_anchor": ([_P, _I, _I, _I, _P, _P, _P], None),
            "rqo_encode_residual_rot": ([_P, _P, _I, _I, _I, _I, _P, _P, _P, _P], None),
            "rqo_encode_residual": ([_P, _P, _I, _I, _I, _I, _P, _P, _P, _P], None),
            "rqo_encode_anchor_rows": ([_P, _I64, _I, _I, _I, _P, _P, _P], None),
            "rqo_encode_residual_rows": ([_P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P], None),
            "rqo_dequant_codes_f64": ([_P, _P, _I, _I, _I, _P], None),
            "rqo_dequant_rows_f64": ([_P, _P, _I64, _I, _I, _I, _P], None),
            "rqo_attention_f64": ([_P, _P, _P, _I64, _P, _P, _I, _D, _P], None),
            "rqo_effective_bits": ([_I, _P, _P, _I, _I, _I], _D),
            "rqo_component_reads": ([_I, _I], _I64),
            "rqo_code_pos": ([_I, _I, _P, _P], None),
            "rqo_m8_scale_encode": ([_F], ctypes.c_uint8),
            "rqo_m8_scale_decode": ([ctypes.c_uint8], _F),
            "rqo_quantize_m8": ([_P, _I, _I, _I, _P, _P, _P], None),
            "rqo_encode_anchor_rows_m8": ([_P, _I64, _I, _I, _I, _P, _P, _P], None),
            "rqo_encode_residual_rot_m8": ([_P, _P, _I, _I, _I, _I, _P, _P, _P, _P], None),
            "rqo_encode_residual_rows_m8": ([_P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P],
                                            None),
            "rqo_dequant_rows_m8_f64": ([_P, _P, _I64, _I, _I, _I, _P], None),
            "rqo_encode_residual_rot_ex": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P],
                                           None),
            "rqo_encode_residual_rows_ex": ([_P, _P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P,
                                             _P], None),
            "rqo_rotate_dense_row": ([_P, _P, _I, _P, _P], None),
            "rqo_rotate_dense_rows": ([_P, _P, _I64, _I, _P, _P], None),
            "rqo_quantize_box": ([_P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P], None),
            "rqo_quantize_box_rows": ([_P, _P, _P, _I64, _I, _I, _I, _P, _P, _P, _P, _P], None),
            "rqo_encode_residual_box": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P,
                                         _P, _P, _P], None),
            "rqo_encode_residual_box_rows": ([_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _P, _P,
                                              _P, _P, _P, _P, _P], None),
        }
        for name, (args, res) in sig.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = res
        _lib = h
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


MAX_D = 256   # the C row functions keep rows of up to 256 channels on the stack


def _check_dim(D: int) -> int:
    """Head dimension accepted by the C row functions: a power of two in
    [32, 256] (the FWHT needs a power of two; rows live in 256-entry stack
    buffers).  Anything else raises before the C code runs."""
    D = int(D)
    if D < 32 or D > MAX_D or D & (D - 1):
        raise ValueError(f"oracle: head_dim {D} is not a power of two in [32, {MAX_D}]")
    return D


# --------------------------------------------------------------------------
# Scalar / row-level entry points (used by the pins)
# --------------------------------------------------------------------------

def f32_to_f16_bits(v: float) -> int:
    return int(lib().rqo_f32_to_f16(float(v)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().rqo_f16_to_f32(int(h)))


def f32_to_bf16_bits(v: float) -> int:
    return int(lib().rqo_f32_to_bf16(float(v)))


def bf16_bits_to_f32(h: int) -> float:
    return float(lib().rqo_bf16_to_f32(int(h)))


def rot_scale(D: int) -> float:
    return float(lib().rqo_rot_scale(D))


def fwht_f32(z: np.ndarray) -> np.ndarray:
    """Normalised Hadamard transform of each row of z (fp32, canonical order)."""
    z = np.array(z, dtype=np.float32, order="C", copy=True)
    D = _check_dim(z.shape[-1])
    flat = z.reshape(-1, D)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib().rqo_fwht_f32(_ptr(row), D)
        flat[r] = row
    return flat.reshape(z.shape)


def fwht_f64(z: np.ndarray) -> np.ndarray:
    z = np.array(z, dtype=np.float64, order="C", copy=True)
    D = _check_dim(z.shape[-1])
    n = z.size // D
    lib().rqo_fwht_rows_f64(_ptr(z), n, D)
    return z


def dot_f32(a: np.ndarray, b: np.ndarray) -> float:
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = np.ascontiguousarray(b, dtype=np.float32)
    return float(lib().rqo_dot_f32(_ptr(a), _ptr(b), a.shape[-1]))


def quantize(z: np.ndarray, bits: int, group: int):
    """Affine-quantise one rotated fp32 row: (words, meta, deq)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    D = _check_dim(z.shape[-1])
    words = np.zeros(D * bits // 32, np.uint32)
    meta = np.zeros(D // group, np.uint32)
    deq = np.zeros(D, np.float32)
    lib().rqo_quantize(_ptr(z), D, bits, group, _ptr(words), _ptr(meta), _ptr(deq))
    return words, meta, deq


M8_BIAS = 18   # exponent bias of the 16-bit-metadata scale byte (rqo.h)


def m8_scale_encode(s: float) -> int:
    """Scale byte (unsigned e5m3) of the 16-bit-metadata variant."""
    return int(lib().rqo_m8_scale_encode(float(s)))


def m8_scale_decode(b: int) -> float:
    return float(lib().rqo_m8_scale_decode(int(b)))


def quantize_m8(z: np.ndarray, bits: int, group: int):
    """Affine-quantise one rotated fp32 row with 16-bit metadata per group:
    (words, meta uint16 [D/group] = scale byte | offset byte << 8, deq)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    D = _check_dim(z.shape[-1])
    words = np.zeros(D * bits // 32, np.uint32)
    meta = np.zeros(D // group, np.uint16)
    deq = np.zeros(D, np.float32)
    lib().rqo_quantize_m8(_ptr(z), D, bits, group, _ptr(words), _ptr(meta), _ptr(deq))
    return words, meta, deq


def encode_residual_rot(z: np.ndarray, ref: np.ndarray, bits: int, group: int,
                        unit_alpha: bool = False):
    """Residual encoder on an already-rotated fp32 row: (words, meta, alpha_bits, zhat)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    ref = np.ascontiguousarray(ref, dtype=np.float32)
    D = _check_dim(z.shape[-1])
    words = np.zeros(D * bits // 32, np.uint32)
    meta = np.zeros(D // group, np.uint32)
    alpha = np.zeros(1, np.uint16)
    zhat = np.zeros(D, np.float32)
    lib().rqo_encode_residual_rot(_ptr(z), _ptr(ref), D, bits, group, int(unit_alpha),
                                  _ptr(words), _ptr(meta), _ptr(alpha), _ptr(zhat))
    return words, meta, int(alpha[0]), zhat


def encode_residual_rot_m8(z: np.ndarray, ref: np.ndarray, bits: int, group: int,
                           unit_alpha: bool = False):
    """encode_residual_rot with 16-bit metadata: (words, meta uint16, alpha_bits, zhat)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    ref = np.ascontiguousarray(ref, dtype=np.float32)
    D = _check_dim(z.shape[-1])
    words = np.zeros(D * bits // 32, np.uint32)
    meta = np.zeros(D // group, np.uint16)
    alpha = np.zeros(1, np.uint16)
    zhat = np.zeros(D, np.float32)
    lib().rqo_encode_residual_rot_m8(_ptr(z), _ptr(ref), D, bits, group, int(unit_alpha),
                                     _ptr(words), _ptr(meta), _ptr(alpha), _ptr(zhat))
    return words, meta, int(alpha[0]), zhat


def encode_residual_rot_ex(z: np.ndarray, ref: np.ndarray, mu: Optional[np.ndarray],
                           bits: int, group: int, unit_alpha: bool = False,
                           meta16: bool = False):
    """Residual encoder with a fixed mean (None: no mean) and either metadata
    form: (words, meta, alpha_bits, zhat)."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    ref = np.ascontiguousarray(ref, dtype=np.float32)
    D = _check_dim(z.shape[-1])
    words = np.zeros(D * bits // 32, np.uint32)
    meta = np.zeros(D // group, np.uint16 if meta16 else np.uint32)
    alpha = np.zeros(1, np.uint16)
    zhat = np.zeros(D, np.float32)
    m = None if mu is None else np.ascontiguousarray(mu, dtype=np.float32)
    lib().rqo_encode_residual_rot_ex(_ptr(z), _ptr(ref), None if m is None else _ptr(m), D, bits,
                                     group, int(unit_alpha), int(meta16), _ptr(words),
                                     _ptr(meta), _ptr(alpha), _ptr(zhat))
    return words, meta, int(alpha[0]), zhat


@functools.lru_cache(maxsize=None)
def code_positions(bits: int, D: int):
    """(word, shift) of every channel of a packed row (rqo_code_pos)."""
    wi = np.zeros(D, np.int64)
    sh = np.zeros(D, np.uint32)
    w = ctypes.c_int()
    s = ctypes.c_int()
    for i in range(D):
        lib().rqo_code_pos(i, bits, ctypes.byref(w), ctypes.byref(s))
        wi[i], sh[i] = w.value, s.value
    return wi, sh


def unpack_codes(words: np.ndarray, bits: int, D: int) -> np.ndarray:
    """Codes of packed rows [..., D*bits/32] -> [..., D] (uint8)."""
    wi, sh = code_positions(bits, D)
    w = np.asarray(words, dtype=np.uint32)
    return ((w[..., wi] >> sh) & np.uint32((1 << bits) - 1)).astype(np.uint8)


def meta_scale_zero(meta: np.ndarray):
    """fp16 (scale, offset) of packed metadata words, as float32 arrays."""
    m = np.asarray(meta, dtype=np.uint32)
    s = (m & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float32)
    z = (m >> 16).astype(np.uint16).view(np.float16).astype(np.float32)
    return s, z


# --------------------------------------------------------------------------
# Layer-side encoder
# --------------------------------------------------------------------------

def encode_side(x: np.ndarray, bits: Sequence[int], group: Sequence[int],
                policy: str = POLICY_LAST, unit_alpha: bool = False, meta16: bool = False,
                mu: Optional[np.ndarray] = None) -> List[Dict[str, np.ndarray]]:
    """Encode every loop of one (layer, K|V) side.

    x: uint16 [L, N, D].  The anchor loop (anchor_loop) is quantised directly;
    every other loop r stores the LS coefficient against its reference's
    reconstruction (alpha = 1 if unit_alpha) and its quantised residual.
    Returns per loop l a dict with 'codes', 'meta', 'alpha' (None for the
    anchor) and 'zhat' (fp32 reconstructed rotated row, the value a chained
    neighbour references).  meta16: 16-bit metadata per group (uint16 meta,
    rqo_quantize_m8) instead of fp16 scale + fp16 offset (uint32 meta).
    mu: optional fp32 [L, N, D] fixed means of the residual loops in the
    rotated domain [RQ App. G.2] (the anchor's entry is not used).
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    L, N, D = x.shape
    _check_dim(D)
    mdt = np.uint16 if meta16 else np.uint32
    enc_anchor = lib().rqo_encode_anchor_rows_m8 if meta16 else lib().rqo_encode_anchor_rows
    enc_resid = lib().rqo_encode_residual_rows_m8 if meta16 else lib().rqo_encode_residual_rows
    out: List[Optional[Dict[str, np.ndarray]]] = [None] * L
    a = anchor_loop(L, policy)
    enc = {"codes": np.zeros((N, D * bits[a] // 32), np.uint32),
           "meta": np.zeros((N, D // group[a]), mdt),
           "alpha": None,
           "zhat": np.zeros((N, D), np.float32)}
    enc_anchor(_ptr(x[a]), N, D, bits[a], group[a], _ptr(enc["codes"]), _ptr(enc["meta"]),
               _ptr(enc["zhat"]))
    out[a] = enc
    for r in encode_order(L, policy):
        ref = out[reference_loop(L, r, policy)]["zhat"]
        enc = {"codes": np.zeros((N, D * bits[r] // 32), np.uint32),
               "meta": np.zeros((N, D // group[r]), mdt),
               "alpha": np.zeros(N, np.uint16),
               "zhat": np.zeros((N, D), np.float32)}
        if mu is None:
            enc_resid(_ptr(x[r]), _ptr(np.ascontiguousarray(ref)), N, D, bits[r], group[r],
                      int(unit_alpha), _ptr(enc["codes"]), _ptr(enc["meta"]),
                      _ptr(enc["alpha"]), _ptr(enc["zhat"]))
        else:
            m = np.ascontiguousarray(mu[r], dtype=np.float32)
            lib().rqo_encode_residual_rows_ex(
                _ptr(x[r]), _ptr(np.ascontiguousarray(ref)), _ptr(m), N, D, bits[r], group[r],
                int(unit_alpha), int(meta16), _ptr(enc["codes"]), _ptr(enc["meta"]),
                _ptr(enc["alpha"]), _ptr(enc["zhat"]))
        out[r] = enc
    return out  # type: ignore[return-value]


def _levels_f64(enc: Dict[str, np.ndarray], bits: int, group: int, D: int) -> np.ndarray:
    """fp64 stored levels of a component (either metadata form, by its dtype)."""
    N = enc["codes"].shape[0]
    out = np.zeros((N, D), np.float64)
    fn = lib().rqo_dequant_rows_m8_f64 if enc["meta"].dtype == np.uint16 else \
        lib().rqo_dequant_rows_f64
    fn(_ptr(enc["codes"]), _ptr(enc["meta"]), N, D, bits, group, _ptr(out))
    return out


def reconstruct_rotated(encs: List[Dict[str, np.ndarray]], loop: int, bits: Sequence[int],
                        group: Sequence[int], policy: str = POLICY_LAST,
                        mu: Optional[np.ndarray] = None) -> np.ndarray:
    """fp64 rotated reconstruction Z^_loop [RQ App. G.2]:
    Z^_anchor = A; Z^_r = alpha~_r * Z^_ref + D(c_r) (+ mu_r, the fixed mean,
    when mu [L, N, D] is given), ref the anchor (shared policies) or the
    neighbour toward the anchor (chained policies), so a chained loop is
    rebuilt from the anchor outwards."""
    L = len(encs)
    a = anchor_loop(L, policy)
    D = encs[a]["zhat"].shape[1]
    z = _levels_f64(encs[a], bits[a], group[a], D)
    if loop == a:
        return z
    path = [loop]
    while reference_loop(L, path[-1], policy) != a:
        path.append(reference_loop(L, path[-1], policy))
    for r in reversed(path):
        al = (encs[r]["alpha"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        z = al[:, None] * z + _levels_f64(encs[r], bits[r], group[r], D)
        if mu is not None:
            z = z + np.asarray(mu[r], np.float64)
    return z


def reconstruct(encs, loop, bits, group, policy=POLICY_LAST, mu=None) -> np.ndarray:
    """fp64 reconstruction in the original domain: X^ = H^T Z^ (H symmetric)."""
    return fwht_f64(reconstruct_rotated(encs, loop, bits, group, policy, mu))


def attention(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, kcur: np.ndarray,
              vcur: np.ndarray, scale: float) -> np.ndarray:
    """fp64 softmax attention of one query over T past rows plus the current token."""
    q = np.ascontiguousarray(q, np.float64)
    khat = np.ascontiguousarray(khat, np.float64)
    vhat = np.ascontiguousarray(vhat, np.float64)
    kcur = np.ascontiguousarray(kcur, np.float64)
    vcur = np.ascontiguousarray(vcur, np.float64)
    D = q.shape[-1]
    T = khat.shape[0]
    out = np.zeros(D, np.float64)
    lib().rqo_attention_f64(_ptr(q), _ptr(khat), _ptr(vhat), T, _ptr(kcur), _ptr(vcur), D,
                            float(scale), _ptr(out))
    return out


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_attention(khat: np.ndarray, vhat: np.ndarray, q_bits: np.ndarray,
                     seq_lens: Sequence[int], kcur_bits: np.ndarray, vcur_bits: np.ndarray,
                     scale: Optional[float] = None) -> np.ndarray:
    """fp64 decode attention for one loop [RQ §4.2 Decode].

    khat, vhat: fp64 [B, H, T, D] reconstructed past keys / values (original
    domain); q_bits, kcur_bits, vcur_bits: bf16 bits [B, H, D]; seq_lens[b]
    past tokens of sequence b.  Returns fp64 [B, H, D]."""
    B, H, T, D = khat.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    q = bf16_bits_to_f64(q_bits)
    kc = bf16_bits_to_f64(kcur_bits)
    vc = bf16_bits_to_f64(vcur_bits)
    out = np.zeros((B, H, D), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            out[b, h] = attention(q[b, h], khat[b, h, :n], vhat[b, h, :n], kc[b, h], vc[b, h],
                                  scale)
    return out


# --------------------------------------------------------------------------
# Dense rotation [RQ §3.3, App. G.1, App. G.2]
# --------------------------------------------------------------------------

def rotate_dense(u: np.ndarray, x: np.ndarray):
    """z = U x for rows x (bf16 bits [n, D]) with U binary16 bits [D, D] (row i
    = output channel i): x is rounded to binary16 and the exact products are
    summed in fp64.  Returns (z fp64 [n, D], bound fp64 [n, D]): every order of
    fp32 accumulation of those products lands within bound of z."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    D = _check_dim(x.shape[-1])
    assert u.shape == (D, D)
    n = x.size // D
    z = np.zeros((n, D), np.float64)
    b = np.zeros((n, D), np.float64)
    lib().rqo_rotate_dense_rows(_ptr(u), _ptr(x), n, D, _ptr(z), _ptr(b))
    return z.reshape(x.shape), b.reshape(x.shape)


def f32_box(z: np.ndarray, bound: np.ndarray):
    """fp32 (lo, hi, mid): lo <= z - bound and hi >= z + bound as fp32 values,
    mid = fp32 rounding of z.  A zero bound on a value exact in fp32 (every
    accumulation order gives exactly z) is a box of one point."""
    mid = z.astype(np.float32)
    lo = np.nextafter((z - bound).astype(np.float32), np.float32(-np.inf))
    hi = np.nextafter((z + bound).astype(np.float32), np.float32(np.inf))
    point = (bound == 0.0) & (mid.astype(np.float64) == z)
    lo = np.where(point, mid, lo)
    hi = np.where(point, mid, hi)
    return (np.ascontiguousarray(lo), np.ascontiguousarray(hi), np.ascontiguousarray(mid))


def quantize_box(lo: np.ndarray, hi: np.ndarray, mid: np.ndarray, bits: int, group: int):
    """Interval quantiser over rows [n, D] (binary16 metadata): (codes, meta,
    deq, meta_ok [n, D/group], code_ok [n, D]); the flags mark the decisions
    every fp32 row inside the box shares."""
    lo, hi, mid = (np.ascontiguousarray(a, dtype=np.float32) for a in (lo, hi, mid))
    D = _check_dim(mid.shape[-1])
    n = mid.size // D
    codes = np.zeros((n, D * bits // 32), np.uint32)
    meta = np.zeros((n, D // group), np.uint32)
    deq = np.zeros((n, D), np.float32)
    mok = np.zeros((n, D // group), np.uint8)
    cok = np.zeros((n, D), np.uint8)
    lib().rqo_quantize_box_rows(_ptr(lo), _ptr(hi), _ptr(mid), n, D, bits, group, _ptr(codes),
                                _ptr(meta), _ptr(deq), _ptr(mok), _ptr(cok))
    return codes, meta, deq, mok.astype(bool), cok.astype(bool)


def encode_side_dense(x: np.ndarray, u: np.ndarray, heads: int, tokens: int,
                      bits: Sequence[int], group: Sequence[int], policy: str = POLICY_LAST,
                      unit_alpha: bool = False, mu: Optional[np.ndarray] = None,
                      meta16: bool = False) -> List[Dict[str, np.ndarray]]:
    """encode_side with the dense rotation of one (layer, K|V) side
    [RQ §3.3, App. G.2]: u binary16 bits [heads, D, D], one matrix per head
    shared by every loop; rows of x [L, N, D] are (b, h, t) with `tokens` rows
    per (b, h); mu as in encode_side.

    The accumulation order of the rotation is not fixed by the pages, so the
    encoder works on the box of fp32 rows that any order can produce
    (rotate_dense's bound): 'codes', 'meta', 'alpha', 'zhat' are those of the
    fp32-rounded exact rotation, and 'code_ok', 'meta_ok', 'alpha_ok' mark the
    decisions that every row of the box shares (a row whose reference is not
    fully determined gets no flag).  The interval form covers binary16
    metadata; with meta16 (16-bit metadata, R22) every rotation must be exact
    (boxes of one point), and the point encoders give the one answer."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    L, N, D = x.shape
    _check_dim(D)
    u = np.ascontiguousarray(u, dtype=np.uint16)
    assert u.shape == (heads, D, D) and N % (heads * tokens) == 0
    head_of = (np.arange(N) // tokens) % heads
    boxes = []
    for l in range(L):
        z = np.zeros((N, D), np.float64)
        bd = np.zeros((N, D), np.float64)
        for h in range(heads):
            rows = np.nonzero(head_of == h)[0]
            zh, bh = rotate_dense(u[h], x[l][rows])
            z[rows], bd[rows] = zh, bh
        boxes.append(f32_box(z, bd))
    if meta16:
        return _encode_points_m8(boxes, bits, group, policy, unit_alpha, mu)
    out: List[Optional[Dict[str, np.ndarray]]] = [None] * L
    a = anchor_loop(L, policy)
    lo, hi, mid = boxes[a]
    codes, meta, deq, mok, cok = quantize_box(lo, hi, mid, bits[a], group[a])
    out[a] = {"codes": codes, "meta": meta, "alpha": None, "zhat": deq,
              "meta_ok": mok, "code_ok": cok, "alpha_ok": None,
              "clean": mok.all(axis=1) & cok.all(axis=1)}
    for r in encode_order(L, policy):
        ref_enc = out[reference_loop(L, r, policy)]
        lo, hi, mid = boxes[r]
        G = D // group[r]
        enc = {"codes": np.zeros((N, D * bits[r] // 32), np.uint32),
               "meta": np.zeros((N, G), np.uint32),
               "alpha": np.zeros(N, np.uint16),
               "zhat": np.zeros((N, D), np.float32)}
        aok = np.zeros(N, np.uint8)
        mok = np.zeros((N, G), np.uint8)
        cok = np.zeros((N, D), np.uint8)
        m = None if mu is None else np.ascontiguousarray(mu[r], dtype=np.float32)
        lib().rqo_encode_residual_box_rows(
            _ptr(lo), _ptr(hi), _ptr(mid), _ptr(np.ascontiguousarray(ref_enc["zhat"])),
            None if m is None else _ptr(m), N, D, bits[r], group[r], int(unit_alpha),
            _ptr(enc["codes"]), _ptr(enc["meta"]), _ptr(enc["alpha"]), _ptr(enc["zhat"]),
            _ptr(aok), _ptr(mok), _ptr(cok))
        ref_clean = ref_enc["clean"]
        enc["alpha_ok"] = aok.astype(bool) & ref_clean
        enc["meta_ok"] = mok.astype(bool) & ref_clean[:, None]
        enc["code_ok"] = cok.astype(bool) & ref_clean[:, None]
        enc["clean"] = enc["alpha_ok"] & enc["meta_ok"].all(axis=1) & enc["code_ok"].all(axis=1)
        out[r] = enc
    return out  # type: ignore[return-value]


def _encode_points_m8(boxes, bits, group, policy, unit_alpha, mu):
    """encode_side_dense with 16-bit metadata on exact rotations."""
    L = len(boxes)
    for lo, hi, mid in boxes:
        if not (np.array_equal(lo, mid) and np.array_equal(hi, mid)):
            raise ValueError("16-bit metadata with a dense rotation needs exact sums")
    N, D = boxes[0][2].shape
    out: List[Optional[Dict[str, np.ndarray]]] = [None] * L
    a = anchor_loop(L, policy)
    z = boxes[a][2]
    enc = {"codes": np.zeros((N, D * bits[a] // 32), np.uint32),
           "meta": np.zeros((N, D // group[a]), np.uint16), "alpha": None,
           "zhat": np.zeros((N, D), np.float32)}
    for n in range(N):
        enc["codes"][n], enc["meta"][n], enc["zhat"][n] = quantize_m8(z[n], bits[a], group[a])
    out[a] = enc
    for r in encode_order(L, policy):
        ref = out[reference_loop(L, r, policy)]["zhat"]
        z = boxes[r][2]
        enc = {"codes": np.zeros((N, D * bits[r] // 32), np.uint32),
               "meta": np.zeros((N, D // group[r]), np.uint16),
               "alpha": np.zeros(N, np.uint16), "zhat": np.zeros((N, D), np.float32)}
        for n in range(N):
            m = None if mu is None else mu[r][n]
            w_, m_, al, zh = encode_residual_rot_ex(z[n], ref[n], m, bits[r], group[r],
                                                    unit_alpha, meta16=True)
            enc["codes"][n], enc["meta"][n], enc["alpha"][n], enc["zhat"][n] = w_, m_, al, zh
        out[r] = enc
    for l in range(L):
        e = out[l]
        e["code_ok"] = np.ones((N, D), bool)
        e["meta_ok"] = np.ones(e["meta"].shape, bool)
        e["alpha_ok"] = None if e["alpha"] is None else np.ones(N, bool)
        e["clean"] = np.ones(N, bool)
    return out


def f16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, np.uint16).view(np.float16).astype(np.float64)


def reconstruct_dense(encs, loop, bits, group, u: np.ndarray, heads: int, tokens: int,
                      policy=POLICY_LAST, mu=None) -> np.ndarray:
    """fp64 reconstruction in the original domain under the dense rotation:
    X^ = U^T Z^ per row, U the row's head matrix [RQ App. G.2]."""
    z = reconstruct_rotated(encs, loop, bits, group, policy, mu)
    N = z.shape[0]
    head_of = (np.arange(N) // tokens) % heads
    uf = f16_bits_to_f64(u)
    out = np.zeros_like(z)
    for h in range(heads):
        rows = head_of == h
        out[rows] = z[rows] @ uf[h]          # row form of U^T z
    return out


def rotate_query_dense(q_bits: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Exact U q of bf16 queries rounded to binary16 (the pages' FP16 inputs):
    q_bits [..., D], u [D, D] binary16 bits -> fp64."""
    qh = f16_bits_to_f64(np.asarray(
        [f32_to_f16_bits(float(v)) for v in bf16_bits_to_f64(q_bits).ravel()],
        np.uint16)).reshape(np.shape(q_bits))
    return qh @ f16_bits_to_f64(u).T


def decode_attention_dense(zk: np.ndarray, zv: np.ndarray, q_bits: np.ndarray,
                           seq_lens: Sequence[int], kcur_bits: np.ndarray,
                           vcur_bits: np.ndarray, uk: np.ndarray, uv: np.ndarray,
                           scale: Optional[float] = None) -> np.ndarray:
    """fp64 decode attention under dense rotations [RQ App. G.2]: scores
    (U_K q~) . Z^_K with q~ the query rounded to binary16, values
    U_V^T sum_t p_t Z^_V,t; the current token's k_cur / v_cur stay in the
    original domain.  zk, zv: fp64 rotated reconstructions [B, H, T, D];
    uk, uv: binary16 bits [H, D, D]; the rest as decode_attention."""
    B, H, T, D = zk.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    kc = bf16_bits_to_f64(kcur_bits)
    vc = bf16_bits_to_f64(vcur_bits)
    out = np.zeros((B, H, D), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            qr = rotate_query_dense(q_bits[b, h], uk[h])
            s = np.concatenate([zk[b, h, :n] @ qr, [bf16_bits_to_f64(q_bits[b, h]) @ kc[b, h]]])
            # the current token's score uses the unrotated query
            s = s * scale
            p = np.exp(s - s.max())
            acc = p[:n] @ zv[b, h, :n]
            o = f16_bits_to_f64(uv[h]).T @ acc + p[n] * vc[b, h]
            out[b, h] = o / p.sum()
    return out


def effective_bits(bits: Sequence[int], group: Sequence[int], D: int, meta_bits: int,
                   residual: bool) -> float:
    L = len(bits)
    b = np.ascontiguousarray(bits, np.int32)
    g = np.ascontiguousarray(group, np.int32)
    return float(lib().rqo_effective_bits(L, _ptr(b), _ptr(g), D, meta_bits, int(residual)))


def component_reads(L: int, chained: bool) -> int:
    return int(lib().rqo_component_reads(L, int(chained)))
