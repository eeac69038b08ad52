"""Seeded synthetic looped-Transformer KV states and queries.

Shared input generator for the tests, the benchmark and the oracle side of
the tests.  It holds none of the method's arithmetic: it only draws numbers.

Every value is a pure function of (seed, layer, side, loop, kind, position),
computed from a counter-based hash (SplitMix64's output function applied to
key + (index + 1) * golden-gamma), so any slice can be generated alone and
CPU and CUDA produce bit-identical bf16 tensors (integer arithmetic, then
IEEE fp64/fp32 multiply-add steps that round identically on both devices).

Distributions (the looped-KV workloads of the ResidualQuant paper, Ouro-1.4B /
Huginn-3.5B shaped):
  N(0,1)  Irwin-Hall: sum of twelve 16-bit uniforms from three hashes,
          centred and divided by 2^16 (variance 1 up to 2^-32).
  U(0,1)  top 24 bits of one hash, (k + 0.5) / 2^24.
  Anchor (final loop)    X_L = c * R0
  Loop r < L (default)   X_r = c * (a_r * R0 + sigma_r * N_r)
  Loop r < L ("tiny")    X_r = a_r * (c * R0) + sigma_r * N_r
  with R0, N_r ~ N(0,1) per (b, h, t, d), a_r ~ U(lo, hi) per (b, h, t),
  c[h, d] = exp(key_scale_std * N(0,1)) for keys and 1 for values.
  Queries q ~ N(0,1) per (b, h, d) per loop; the current token of a decode
  step is position t = T of the same recipe.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
T_SPACE = 1 << 21          # index space reserved per (b, h) for token positions

KIND_R, KIND_N, KIND_A, KIND_C, KIND_Q = 1, 2, 3, 4, 5
SIDE_K, SIDE_V = 0, 1


def _s64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix64_py(z: int) -> int:
    """SplitMix64 output function on a Python int (reference form)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def hash_py(key: int, idx: int) -> int:
    return mix64_py((key + (idx + 1) * GAMMA) & MASK64)


def stream_key(seed: int, layer: int, side: int, loop: int, kind: int) -> int:
    tag = (((layer * 64 + loop) * 4 + side) * 16 + kind)
    return mix64_py(((seed + 1) * GAMMA) ^ mix64_py(tag))


def _srl(z: torch.Tensor, k: int) -> torch.Tensor:
    return (z >> k) & ((1 << (64 - k)) - 1)


def hash_t(key: int, idx: torch.Tensor) -> torch.Tensor:
    """Tensor form of hash_py: int64 tensors holding the 64 hash bits."""
    z = (idx + 1) * _s64(GAMMA) + _s64(key)
    z = (z ^ _srl(z, 30)) * _s64(M1)
    z = (z ^ _srl(z, 27)) * _s64(M2)
    return z ^ _srl(z, 31)


def normal_t(key: int, idx: torch.Tensor) -> torch.Tensor:
    """Irwin-Hall N(0,1) samples (float64, exact multiples of 2^-16)."""
    s = torch.zeros_like(idx)
    for j in range(3):
        h = hash_t(key, idx * 3 + j)
        for k in range(4):
            s = s + (_srl(h, 16 * k) & 0xFFFF)
    return (s - 393210).to(torch.float64) / 65536.0


def uniform_t(key: int, idx: torch.Tensor) -> torch.Tensor:
    h = hash_t(key, idx)
    return (_srl(h, 40).to(torch.float64) + 0.5) / float(1 << 24)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic looped-KV workload."""
    name: str
    loops: int                 # L; loop L-1 (0-based) is the final-loop anchor
    batch: int
    heads: int                 # KV heads (MHA: query heads = KV heads)
    head_dim: int
    tokens: int                # past tokens T
    bits: Tuple[int, ...]      # per loop, [L-1] = anchor
    group: Tuple[int, ...]
    sigma: Tuple[float, ...]   # noise std of loops 0..L-2
    a_range: Tuple[float, float]
    seed: int
    layers: int = 1
    key_scale_std: float = 0.5
    recipe: str = "default"    # "default" or "tiny"
    batch0: int = 0            # global index of batch row 0 (a slice of a larger batch)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _linspace(a: float, b: float, n: int) -> Tuple[float, ...]:
    return tuple(a + (b - a) * i / (n - 1) for i in range(n))


# The five workloads of the method's hot path (tiny reference, Ouro-like
# layer, Ouro-like 16k decode step, prefill-sized quantize, Huginn-like deep
# recurrence).
WORKLOADS = {
    "tiny": Workload("tiny", 2, 1, 2, 64, 256, (2, 4), (32, 32), (0.3,), (0.8, 1.2), 0,
                     recipe="tiny"),
    "ouro_layer": Workload("ouro_layer", 4, 8, 16, 128, 4096, (2, 2, 2, 4), (32,) * 4,
                           (0.35, 0.25, 0.15), (0.8, 1.2), 1),
    "ouro_16k": Workload("ouro_16k", 4, 16, 16, 128, 16384, (4, 2, 2, 4), (32,) * 4,
                         (0.35, 0.25, 0.15), (0.8, 1.2), 2, layers=24),
    "quantize_prefill": Workload("quantize_prefill", 4, 4, 16, 128, 16384, (2, 2, 2, 4),
                                 (32,) * 4, (0.35, 0.25, 0.15), (0.8, 1.2), 3),
    "huginn_deep": Workload("huginn_deep", 8, 32, 40, 128, 8192, (2,) * 7 + (4,), (64,) * 8,
                            _linspace(0.4, 0.1, 7), (0.7, 1.3), 4),
}


def key_channel_scale(w: Workload, layer: int) -> torch.Tensor:
    """c[h, d] = exp(key_scale_std * N(0,1)), float32 (computed on the host)."""
    idx = torch.arange(w.heads * w.head_dim, dtype=torch.int64)
    n = normal_t(stream_key(w.seed, layer, SIDE_K, 0, KIND_C), idx)
    return torch.exp(w.key_scale_std * n).to(torch.float32).reshape(w.heads, w.head_dim)


def _row_index(w: Workload, b: torch.Tensor, h: torch.Tensor, t: torch.Tensor) -> torch.Tensor:
    b = b + w.batch0
    return (b[:, None, None] * w.heads + h[None, :, None]) * T_SPACE + t[None, None, :]


def partition(w: Workload, rank: int, world: int) -> Workload:
    """Rank `rank`'s share of w's batch when `world` ranks split it: rows
    [rank*B/world, (rank+1)*B/world) (B = w.batch), as a workload whose values
    are exactly those rows of w (the generator indexes global rows)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    lo = rank * w.batch // world
    hi = (rank + 1) * w.batch // world
    return w.replace(batch0=w.batch0 + lo, batch=hi - lo)


def kv(w: Workload, layer: int, side: int, loop: int, b: Sequence[int], h: Sequence[int],
       t0: int, t1: int, device="cpu", cscale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 [len(b), len(h), t1-t0, D] states of `loop` for the selected rows
    (b: batch rows of w, 0 .. w.batch-1)."""
    dev = torch.device(device)
    bt = torch.as_tensor(list(b), dtype=torch.int64, device=dev)
    ht = torch.as_tensor(list(h), dtype=torch.int64, device=dev)
    tt = torch.arange(t0, t1, dtype=torch.int64, device=dev)
    D = w.head_dim
    rows = _row_index(w, bt, ht, tt)                                   # [b, h, t]
    eidx = rows[..., None] * D + torch.arange(D, dtype=torch.int64, device=dev)
    r0 = normal_t(stream_key(w.seed, layer, side, 0, KIND_R), eidx).to(torch.float32)
    if side == SIDE_K:
        c = (cscale if cscale is not None else key_channel_scale(w, layer)).to(dev)
        c = c[ht][None, :, None, :]
    else:
        c = None
    anchor = w.loops - 1
    if loop == anchor:
        x = r0 * c if c is not None else r0
        return x.to(torch.bfloat16)
    a_lo, a_hi = w.a_range
    a = a_lo + (a_hi - a_lo) * uniform_t(stream_key(w.seed, layer, side, loop, KIND_A), rows)
    a = a.to(torch.float32)[..., None]
    nz = normal_t(stream_key(w.seed, layer, side, loop, KIND_N), eidx).to(torch.float32)
    sig = torch.tensor(w.sigma[loop], dtype=torch.float32, device=dev)
    if w.recipe == "tiny":
        base = r0 * c if c is not None else r0
        x = a * base + sig * nz
    else:
        x = a * r0 + sig * nz
        if c is not None:
            x = x * c
    return x.to(torch.bfloat16)


def query(w: Workload, layer: int, loop: int, device="cpu") -> torch.Tensor:
    """bf16 [B, H, D] query of one decode step for `loop`."""
    dev = torch.device(device)
    idx = torch.arange(w.batch * w.heads * w.head_dim, dtype=torch.int64, device=dev)
    idx = idx + w.batch0 * w.heads * w.head_dim
    n = normal_t(stream_key(w.seed, layer, SIDE_K, loop, KIND_Q), idx).to(torch.float32)
    return n.reshape(w.batch, w.heads, w.head_dim).to(torch.bfloat16)


def all_rows(w: Workload):
    return range(w.batch), range(w.heads)


def kv_full(w: Workload, layer: int, side: int, loop: int, t0: int, t1: int,
            device="cpu", chunk_b: int = 1) -> torch.Tensor:
    """bf16 [B, H, t1-t0, D] for every (b, h), generated chunk by chunk."""
    cs = key_channel_scale(w, layer) if side == SIDE_K else None
    parts = []
    for b0 in range(0, w.batch, chunk_b):
        bs = range(b0, min(w.batch, b0 + chunk_b))
        parts.append(kv(w, layer, side, loop, bs, range(w.heads), t0, t1, device, cs))
    return torch.cat(parts, 0)


def current_token(w: Workload, layer: int, side: int, loop: int, device="cpu") -> torch.Tensor:
    """bf16 [B, H, D]: the decode step's own token (position T) for `loop`."""
    return kv_full(w, layer, side, loop, w.tokens, w.tokens + 1, device)[:, :, 0, :]


def bits_of(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def seq_lens_ragged(w: Workload, min_frac: float = 0.5) -> list:
    """Deterministic ragged past lengths in [min_frac*T, T] (sequence 0 gets T)."""
    out = []
    key = stream_key(w.seed, 0, 0, 0, 15)
    for b in range(w.batch0, w.batch0 + w.batch):
        u = (hash_py(key, b) >> 40) / float(1 << 24)
        n = w.tokens if b == 0 else int(math.floor(w.tokens * (min_frac + (1 - min_frac) * u)))
        out.append(max(0, min(w.tokens, n)))
    return out
