"""Test harness: builds packed caches through the C ABI and the matching
oracle encodings from the same seeded inputs.

Inputs come from residual_bit_kv_b200.synth (bit-identical on CPU and CUDA);
expected values come only from the oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle
import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth

SIDES = (synth.SIDE_K, synth.SIDE_V)


POLICY_CODES = {"last": L.RQ_POLICY_LAST_LOOP, "next": L.RQ_POLICY_NEXT_LOOP,
                "first": L.RQ_POLICY_FIRST_LOOP, "previous": L.RQ_POLICY_PREVIOUS_LOOP}


def policy_code(policy: str) -> int:
    return POLICY_CODES[policy]


def layout_of(w: synth.Workload, policy: str = "last", layers: Optional[int] = None,
              max_tokens: Optional[int] = None, unit_alpha: bool = False,
              meta16: bool = False) -> L.rq_layout:
    flags = (L.RQ_FLAG_UNIT_ALPHA if unit_alpha else 0) | (L.RQ_FLAG_META16 if meta16 else 0)
    return L.make_layout(layers or w.layers, w.loops, w.batch, w.heads, w.head_dim,
                         max_tokens or (w.tokens + 1), w.bits, w.group, policy_code(policy),
                         flags)


def append_order(w: synth.Workload, policy: str) -> List[int]:
    """Anchor first, then the other loops away from it (as a chain requires)."""
    a = oracle.anchor_loop(w.loops, policy)
    return [a] + oracle.encode_order(w.loops, policy)


@dataclasses.dataclass
class GpuCache:
    w: synth.Workload
    policy: str
    layout: L.rq_layout
    cache: L.rq_cache
    kbuf: torch.Tensor
    vbuf: torch.Tensor
    inputs: Dict  # (layer, side, loop) -> bf16 [B, H, T, D] cuda tensor (if kept)
    unit_alpha: bool = False
    meta16: bool = False
    means: Optional[Dict] = None   # side -> fp32 [layers, loops, H, D] cuda tensor
    rot: Optional[Dict] = None     # side -> binary16 [layers, H, D, D] cuda tensor (or None)


def build_gpu_cache(w: synth.Workload, policy: str = "last", layers: Sequence[int] = (0,),
                    keep_inputs: bool = True, tokens: Optional[int] = None,
                    max_tokens: Optional[int] = None, append_chunks: Optional[Sequence[int]] = None,
                    fused: bool = False, unit_alpha: bool = False,
                    gen_device: str = "cuda", meta16: bool = False,
                    means_seed: Optional[int] = None,
                    rotations: Optional[Dict] = None) -> GpuCache:
    """Generates every loop's K/V on the GPU and quantise-appends them through
    the C ABI in the order the policy requires (fused: every loop and both
    sides of a chunk in one rq_quantize_append_loops call).  append_chunks
    splits the token range into consecutive appends (e.g. prefill then
    single tokens).  gen_device "cpu" draws the inputs on the host and copies
    them over (no generator kernels on the GPU)."""
    T = w.tokens if tokens is None else tokens
    lay = layout_of(w, policy, layers=max(layers) + 1, max_tokens=max_tokens, unit_alpha=unit_alpha,
                    meta16=meta16)
    nbytes = L.rq_cache_bytes(lay)
    assert nbytes > 0
    kbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    vbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    cache = L.rq_cache_bind(lay, kbuf, vbuf)
    means = None
    if means_seed is not None:
        g = torch.Generator().manual_seed(means_seed)
        means = {side: (torch.randn(lay.num_layers, w.loops, w.heads, w.head_dim, generator=g) *
                        0.5).to("cuda") for side in SIDES}
        L.rq_cache_set_means(cache, means[0], means[1])
    if rotations is not None:
        L.rq_cache_set_rotations(cache, rotations.get(0), rotations.get(1))
    inputs = {}
    bounds = [0] + list(np.cumsum(append_chunks)) if append_chunks else [0, T]
    assert bounds[-1] == T
    for layer in layers:
        if fused:
            xs = {(side, loop): synth.kv_full(w, layer, side, loop, 0, T, device=gen_device,
                                              chunk_b=4).to("cuda")
                  for side in SIDES for loop in range(w.loops)}
            for a, b in zip(bounds[:-1], bounds[1:]):
                if b == a:
                    continue
                xk, xv = (torch.stack([xs[(side, loop)][:, :, a:b] for loop in range(w.loops)])
                          .contiguous() for side in SIDES)
                L.rq_quantize_append_loops(cache, layer, xk, xv, a, b - a)
            if keep_inputs:
                for (side, loop), x in xs.items():
                    inputs[(layer, side, loop)] = x
            del xs
            continue
        for side in SIDES:
            xs = {loop: synth.kv_full(w, layer, side, loop, 0, T, device=gen_device,
                                      chunk_b=4).to("cuda")
                  for loop in range(w.loops)}
            for a, b in zip(bounds[:-1], bounds[1:]):
                if b == a:
                    continue
                for loop in append_order(w, policy):
                    x = xs[loop][:, :, a:b].contiguous()
                    if loop == oracle.anchor_loop(w.loops, policy):
                        L.rq_quantize_anchor(cache, layer, side, x, a, b - a)
                    else:
                        L.rq_quantize_append_residual(cache, layer, side, loop, x, a, b - a)
            if keep_inputs:
                for loop, x in xs.items():
                    inputs[(layer, side, loop)] = x
            del xs
    torch.cuda.synchronize()
    return GpuCache(w, policy, lay, cache, kbuf, vbuf, inputs, unit_alpha, meta16, means,
                    rotations)


def gpu_component(gc: GpuCache, layer: int, side: int, loop: int,
                  bsel: Optional[Sequence[int]] = None,
                  hsel: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Packed arrays of one component, unblocked from the storage records into
    numpy [B, H, token_stride, ...] arrays (or [len(bsel), len(hsel), ...] for
    a selection, copying only those rows off the device)."""
    c = gc.cache
    w = gc.w
    buf = gc.kbuf if side == synth.SIDE_K else gc.vbuf
    ts = c.token_stride
    blk = L.RQ_BLOCK_TOKENS
    nb = ts // blk
    rb = c.rec_bytes[loop]
    D = w.head_dim
    W = D * w.bits[loop] // 32
    G = D // w.group[loop]
    base = layer * c.layer_bytes + c.comp_off[loop]
    bsel = list(range(w.batch)) if bsel is None else list(bsel)
    hsel = list(range(w.heads)) if hsel is None else list(hsel)
    rows = [b * w.heads + h for b in bsel for h in hsel]
    allrec = buf[base: base + w.batch * w.heads * nb * rb].view(w.batch * w.heads, nb * rb)
    recs = allrec[rows].cpu().numpy().reshape(len(rows) * nb, rb)
    shp = (len(bsel), len(hsel), ts)
    mb = 2 if gc.meta16 else 4
    codes = recs[:, : blk * W * 4].copy().view(np.uint32).reshape(*shp, W)
    meta = recs[:, blk * W * 4: blk * (W * 4 + G * mb)].copy().view(
        np.uint16 if gc.meta16 else np.uint32).reshape(*shp, G)
    out = {"codes": codes, "meta": meta, "alpha": None}
    if loop != oracle.anchor_loop(w.loops, gc.policy):
        a0 = blk * (W * 4 + G * mb)
        out["alpha"] = recs[:, a0: a0 + blk * 2].copy().view(np.uint16).reshape(*shp)
    return out


def oracle_encode(w: synth.Workload, layer: int, side: int, bsel: Sequence[int],
                  hsel: Sequence[int], t0: int, t1: int, policy: str = "last",
                  x_loops: Optional[List[np.ndarray]] = None, unit_alpha: bool = False,
                  meta16: bool = False, means: Optional[Dict] = None):
    """Oracle encodings of the selected rows.  Returns (encs, x) where
    x is uint16 [L, nb*nh*(t1-t0), D] (means: the cache's fixed means)."""
    if x_loops is None:
        cs = synth.key_channel_scale(w, layer) if side == synth.SIDE_K else None
        x_loops = [synth.bits_of(synth.kv(w, layer, side, loop, bsel, hsel, t0, t1, "cpu", cs))
                   .reshape(-1, w.head_dim) for loop in range(w.loops)]
    x = np.stack(x_loops)
    return oracle.encode_side(x, w.bits, w.group, policy, unit_alpha, meta16,
                              mu=mean_rows(w, layer, side, bsel, hsel, t1 - t0, means)), x


def mean_rows(w: synth.Workload, layer: int, side: int, bsel: Sequence[int],
              hsel: Sequence[int], T: int, means: Optional[Dict]) -> Optional[np.ndarray]:
    """The fixed means expanded to the oracle's rows (b, h, t): [L, N, D]."""
    if means is None:
        return None
    m = means[side][layer].cpu().numpy().astype(np.float32)   # [L, H, D]
    rows = [m[:, h] for b in bsel for h in hsel for _ in range(T)]
    return np.ascontiguousarray(np.stack(rows, axis=1))


def assert_component_equal(gpu: Dict[str, np.ndarray], enc: Dict[str, np.ndarray], shape,
                           what: str) -> None:
    """Bit-exact comparison of codes, metadata and LS coefficients."""
    for key in ("codes", "meta", "alpha"):
        g = gpu[key]
        o = enc[key]
        if o is None:
            assert g is None
            continue
        g = np.ascontiguousarray(g).reshape(o.shape)
        bad = np.count_nonzero(g != o)
        assert bad == 0, f"{what} {key}: {bad} of {o.size} words differ"


def decode_inputs(w: synth.Workload, layer: int, loop: int, device="cuda"):
    """q, k_cur, v_cur of one decode call on the GPU, drawn on `device`."""
    q = synth.query(w, layer, loop, device)
    kc = synth.current_token(w, layer, synth.SIDE_K, loop, device)
    vc = synth.current_token(w, layer, synth.SIDE_V, loop, device)
    return tuple(t.contiguous().to("cuda") for t in (q, kc, vc))


class Workspace:
    def __init__(self, layout: L.rq_layout, max_seq_len: int):
        self.bytes = L.rq_decode_workspace_bytes(layout, max_seq_len)
        assert self.bytes > 0
        self.buf = torch.empty(self.bytes, dtype=torch.uint8, device="cuda")
        L.rq_decode_workspace_init(self.buf, self.bytes)


def gpu_decode(gc: GpuCache, layer: int, loop: int, seq_lens: Sequence[int], max_seq_len: int,
               ws: Optional[Workspace] = None, scale: float = 0.0, gen_device: str = "cuda"):
    w = gc.w
    q, kc, vc = decode_inputs(w, layer, loop, gen_device)
    sl = torch.tensor(list(seq_lens), dtype=torch.int32, device="cuda")
    out = torch.empty(w.batch, w.heads, w.head_dim, dtype=torch.float32, device="cuda")
    ws = ws or Workspace(gc.layout, max_seq_len)
    L.rq_decode_attention(gc.cache, layer, loop, q, sl, max_seq_len, kc, vc, scale, out, ws.buf,
                          ws.bytes)
    torch.cuda.synchronize()
    status = L.rq_workspace_error(ws.buf, ws.bytes)
    return out.cpu().numpy().astype(np.float64), status


def oracle_decode(w: synth.Workload, layer: int, loop: int, bsel: Sequence[int],
                  hsel: Sequence[int], seq_lens: Sequence[int], policy: str = "last",
                  inputs: Optional[Dict] = None, scale: Optional[float] = None,
                  unit_alpha: bool = False, meta16: bool = False,
                  means: Optional[Dict] = None) -> np.ndarray:
    """fp64 oracle decode for the selected (b, h): [len(bsel), len(hsel), D]."""
    T = max(int(seq_lens[b]) for b in bsel)
    D = w.head_dim
    outs = []
    rec = {}
    for side in SIDES:
        xl = None
        if inputs is not None:
            xl = [synth.bits_of(inputs[(layer, side, l)][list(bsel)][:, list(hsel), :T].cpu())
                  .reshape(-1, D) for l in range(w.loops)]
        encs, _ = oracle_encode(w, layer, side, bsel, hsel, 0, T, policy, xl, unit_alpha, meta16,
                                means)
        rec[side] = oracle.reconstruct(encs, loop, w.bits, w.group, policy,
                                       mean_rows(w, layer, side, bsel, hsel, T, means)).reshape(
            len(bsel), len(hsel), T, D)
    q = synth.bits_of(synth.query(w, layer, loop)).reshape(w.batch, w.heads, D)
    kc = synth.bits_of(synth.current_token(w, layer, synth.SIDE_K, loop))
    vc = synth.bits_of(synth.current_token(w, layer, synth.SIDE_V, loop))
    bi, hi = np.ix_(list(bsel), list(hsel))
    return oracle.decode_attention(rec[0], rec[1], q[bi, hi], [seq_lens[b] for b in bsel],
                                   kc[bi, hi], vc[bi, hi], scale)


def attn_tolerance(ref: np.ndarray) -> float:
    """max-abs error bound: 2e-3 * max|out| (per the method's parity target)."""
    return 2e-3 * float(np.max(np.abs(ref)))
