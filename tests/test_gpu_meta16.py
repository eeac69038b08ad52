"""16-bit metadata per group (RQ_FLAG_META16) through the C ABI vs the
oracle: bit-exact codes, metadata bytes and LS coefficients (per-loop and
fused appends, every policy); decode attention within 2e-3 * max|out| on the
compiled layouts and on the generic kernel."""
import numpy as np
import pytest

import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import (SIDES, Workspace, assert_component_equal, attn_tolerance,
                        build_gpu_cache, gpu_component, gpu_decode, oracle_decode, oracle_encode)

pytestmark = pytest.mark.gpu


def _check_components(gc, T, bsel, hsel):
    w = gc.w
    for side in SIDES:
        encs, _ = oracle_encode(w, 0, side, bsel, hsel, 0, T, gc.policy,
                                x_loops=None if not gc.inputs else
                                [synth.bits_of(gc.inputs[(0, side, l)][bsel][:, hsel, :T].cpu())
                                 .reshape(-1, w.head_dim) for l in range(w.loops)],
                                unit_alpha=gc.unit_alpha, meta16=True)
        for loop in range(w.loops):
            g = gpu_component(gc, 0, side, loop, bsel, hsel)
            g = {k: (None if v is None else v[:, :, :T]) for k, v in g.items()}
            assert g["meta"].dtype == np.uint16
            assert_component_equal(g, encs[loop], None, f"meta16 side {side} loop {loop}")


@pytest.mark.parametrize("policy", ["last", "next", "first", "previous"])
@pytest.mark.parametrize("fused", [False, True])
def test_meta16_append_bit_exact(cuda_dev, policy, fused):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=333)
    gc = build_gpu_cache(w, policy=policy, fused=fused, meta16=True, append_chunks=[300, 1, 32])
    _check_components(gc, 333, [0, 1], [0, 1, 2])


def test_meta16_groups_and_widths(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=200, bits=(4, 2, 2, 4),
                                              group=(16, 64, 128, 32))
    for fused in (False, True):
        gc = build_gpu_cache(w, fused=fused, meta16=True)
        _check_components(gc, 200, [0, 1], [0, 1])


def test_meta16_head_dim_64(cuda_dev):
    w = synth.WORKLOADS["tiny"]
    gc = build_gpu_cache(w, meta16=True)
    _check_components(gc, w.tokens, [0], list(range(w.heads)))


def _check_decode(gc, seq_lens, max_seq_len, loops=None):
    w = gc.w
    ws = Workspace(gc.layout, max_seq_len)
    for loop in (range(w.loops) if loops is None else loops):
        out, status = gpu_decode(gc, 0, loop, seq_lens, max_seq_len, ws)
        assert status == L.RQ_OK
        ref = oracle_decode(w, 0, loop, list(range(w.batch)), list(range(w.heads)), seq_lens,
                            gc.policy, gc.inputs or None, unit_alpha=gc.unit_alpha, meta16=True)
        err = np.max(np.abs(out - ref))
        assert err <= attn_tolerance(ref), (loop, err, attn_tolerance(ref))


@pytest.mark.parametrize("policy", ["last", "next", "first", "previous"])
def test_meta16_decode_compiled_layouts(cuda_dev, policy):
    """[2,2,2,4] / [4,2,2,2] g 32 at D 128: the compiled (fast) kernels."""
    bits = (2, 2, 2, 4) if policy in ("last", "next") else (4, 2, 2, 2)
    w = synth.WORKLOADS["ouro_layer"].replace(batch=3, heads=2, tokens=700, bits=bits)
    gc = build_gpu_cache(w, policy=policy, meta16=True)
    _check_decode(gc, [700, 0, 129], 700)


def test_meta16_decode_generic_kernel(cuda_dev):
    """Mixed groups (not compiled): the generic decode kernel."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=300, bits=(4, 2, 2, 4),
                                              group=(16, 64, 128, 32))
    gc = build_gpu_cache(w, meta16=True)
    _check_decode(gc, [300, 77], 300)


def test_meta16_storage_halves_metadata():
    """Record bytes: codes + 2 bytes per group (+ 2 for alpha)."""
    w = synth.WORKLOADS["ouro_layer"]
    from rq_harness import layout_of
    l16 = layout_of(w, meta16=True, layers=1)
    l32 = layout_of(w, layers=1)
    per_tok = lambda mb: sum((128 * b // 32) * 4 + (128 // g) * mb + (2 if r != w.loops - 1 else 0)
                             for r, (b, g) in enumerate(zip(w.bits, w.group)))
    T = -(-(w.tokens + 1) // 64) * 64
    assert L.rq_layer_bytes(l16) >= w.batch * w.heads * T * per_tok(2)
    assert L.rq_layer_bytes(l32) - L.rq_layer_bytes(l16) == w.batch * w.heads * T * (
        per_tok(4) - per_tok(2))


def _sampled_full(gc, bsel, hsel, loops):
    """Sampled (batch, head) units at full size: every stored bit of both
    sides, and the decode of `loops` against the oracle."""
    w = gc.w
    T = w.tokens
    for side in SIDES:
        encs, _ = oracle_encode(w, 0, side, bsel, hsel, 0, T, gc.policy, meta16=True)
        for loop in range(w.loops):
            g = gpu_component(gc, 0, side, loop, bsel, hsel)
            g = {k: (None if v is None else v[:, :, :T]) for k, v in g.items()}
            assert_component_equal(g, encs[loop], None, f"meta16 full side {side} loop {loop}")
    ws = Workspace(gc.layout, T)
    for loop in loops:
        out, status = gpu_decode(gc, 0, loop, [T] * w.batch, T, ws)
        assert status == L.RQ_OK
        ref = oracle_decode(w, 0, loop, bsel, hsel, [T] * w.batch, gc.policy, meta16=True)
        got = out[np.ix_(bsel, hsel)]
        err = float(np.max(np.abs(got - ref)))
        assert err <= attn_tolerance(ref), (loop, err, attn_tolerance(ref))


def test_meta16_ouro_16k_full_size(cuda_dev):
    """16k decode workload (batch 16, 16 heads, 16384 tokens, bits [4,2,2,4],
    g 32) stored with 16-bit metadata through the fused all-loops append, in
    the benchmark's launch configuration (capacity T+16): sampled units."""
    import torch
    w = synth.WORKLOADS["ouro_16k"]
    gc = build_gpu_cache(w, keep_inputs=False, max_tokens=w.tokens + 16, fused=True, meta16=True)
    _sampled_full(gc, [0, 15], [3, 12], range(w.loops))
    del gc
    torch.cuda.empty_cache()


def test_meta16_prefill_full_size(cuda_dev):
    """Prefill workload (batch 4, 16 heads, 16384 tokens, INT2 residuals)
    with 16-bit metadata, per-loop appends: sampled units, every bit."""
    import torch
    w = synth.WORKLOADS["quantize_prefill"]
    gc = build_gpu_cache(w, keep_inputs=False, max_tokens=w.tokens, meta16=True)
    _sampled_full(gc, [0, 3], [0, 7, 15], [0, 3])
    del gc
    torch.cuda.empty_cache()
