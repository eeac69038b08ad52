"""Parity at the benchmark workloads' full sizes, in the launch configuration
bench.py times (capacity T+16, every sequence at T past tokens), on sampled
(batch, head) units the oracle computes one by one -- and, for the prefill
workload, every stored code."""
import numpy as np
import pytest
import torch

import oracle
import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import (SIDES, Workspace, assert_component_equal, attn_tolerance, build_gpu_cache,
                        gpu_component, gpu_decode, oracle_decode, oracle_encode)

pytestmark = pytest.mark.gpu


def _sampled_codes_equal(gc, layer, bsel, hsel, policy):
    w = gc.w
    for side in SIDES:
        encs, _ = oracle_encode(w, layer, side, bsel, hsel, 0, w.tokens, policy)
        for loop in range(w.loops):
            g = gpu_component(gc, layer, side, loop, bsel, hsel)
            g = {k: (None if v is None else v[:, :, :w.tokens]) for k, v in g.items()}
            assert_component_equal(g, encs[loop], None, f"layer {layer} side {side} loop {loop}")


def _sampled_decode_close(gc, layer, bsel, hsel, policy, loops=None):
    w = gc.w
    T = w.tokens
    ws = Workspace(gc.layout, T)
    for loop in (range(w.loops) if loops is None else loops):
        out, status = gpu_decode(gc, layer, loop, [T] * w.batch, T, ws)
        assert status == L.RQ_OK
        ref = oracle_decode(w, layer, loop, bsel, hsel, [T] * w.batch, policy)
        got = out[np.ix_(bsel, hsel)]
        err = float(np.max(np.abs(got - ref)))
        assert err <= attn_tolerance(ref), (loop, err)


def test_ouro_layer_full_size(cuda_dev):
    """Ouro-like layer: 4 loops, batch 8, 16 heads, 4096 tokens."""
    w = synth.WORKLOADS["ouro_layer"]
    gc = build_gpu_cache(w, keep_inputs=False, max_tokens=w.tokens + 16)
    bsel, hsel = [0, 7], [0, 9, 15]
    _sampled_codes_equal(gc, 0, bsel, hsel, "last")
    _sampled_decode_close(gc, 0, bsel, hsel, "last")


def test_ouro_16k_step_layers_full_size(cuda_dev):
    """16k decode workload: batch 16, 16 heads, 16384 tokens, bits [4,2,2,4];
    layer 0 and a later layer (distinct data per layer)."""
    w = synth.WORKLOADS["ouro_16k"]
    for layer in (0, 17):
        gc = build_gpu_cache(w, layers=(layer,), keep_inputs=False, max_tokens=w.tokens + 16)
        bsel, hsel = [0, 15], [3, 12]
        _sampled_codes_equal(gc, layer, bsel, hsel, "last")
        _sampled_decode_close(gc, layer, bsel, hsel, "last")
        del gc
        torch.cuda.empty_cache()


def test_prefill_quantize_every_code(cuda_dev):
    """Prefill workload (batch 4, 16 heads, 16384 tokens, INT2 residuals, g 32):
    every stored code, scale, offset and alpha of both sides is bit-exact
    (2 x 402,653,184 residual codes)."""
    w = synth.WORKLOADS["quantize_prefill"]
    gc = build_gpu_cache(w, keep_inputs=True, max_tokens=w.tokens)
    total = 0
    for side in SIDES:
        xl = [synth.bits_of(gc.inputs[(0, side, l)].cpu()).reshape(-1, w.head_dim)
              for l in range(w.loops)]
        encs = oracle.encode_side(np.stack(xl), w.bits, w.group)
        for loop in range(w.loops):
            g = gpu_component(gc, 0, side, loop)
            assert_component_equal(g, encs[loop], None, f"side {side} loop {loop}")
            if loop != w.loops - 1:
                total += encs[loop]["codes"].size * (32 // w.bits[loop])
    assert total == 2 * 3 * 4 * 16 * 16384 * 128


@pytest.mark.parametrize("policy", ["last", "next"])
def test_huginn_deep_full_size(cuda_dev, policy):
    """Deep recurrence: 8 loops, batch 32, 40 heads, 8192 tokens, g 64, shared
    anchor and the chained (Next-loop) ablation."""
    w = synth.WORKLOADS["huginn_deep"]
    gc = build_gpu_cache(w, policy=policy, keep_inputs=False, max_tokens=w.tokens + 16)
    bsel, hsel = [0, 31], [0, 39]
    _sampled_codes_equal(gc, 0, bsel, hsel, policy)
    _sampled_decode_close(gc, 0, bsel, hsel, policy, loops=[0, 3, 6, 7])
    del gc
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_ouro_16k_layer0_every_unit(cuda_dev):
    """16k decode workload, layer 0 in full: every stored code and scale of both
    sides, and the decode output of every (batch, head) for all four loops, in
    the launch configuration the benchmark times (capacity T+16, T past tokens)."""
    w = synth.WORKLOADS["ouro_16k"]
    T, D = w.tokens, w.head_dim
    gc = build_gpu_cache(w, layers=(0,), keep_inputs=True, max_tokens=T + 16)
    ws = Workspace(gc.layout, T)
    outs = {}
    for loop in range(w.loops):
        out, status = gpu_decode(gc, 0, loop, [T] * w.batch, T, ws)
        assert status == L.RQ_OK
        outs[loop] = out
    hsel = list(range(w.heads))
    q = synth.bits_of(torch.stack([synth.query(w, 0, l) for l in range(w.loops)]))
    kc = [synth.bits_of(synth.current_token(w, 0, synth.SIDE_K, l)) for l in range(w.loops)]
    vc = [synth.bits_of(synth.current_token(w, 0, synth.SIDE_V, l)) for l in range(w.loops)]
    units = 0
    for b0 in range(0, w.batch, 4):
        bsel = list(range(b0, b0 + 4))
        encs = {}
        for side in SIDES:
            xl = [synth.bits_of(gc.inputs[(0, side, l)][bsel].cpu()).reshape(-1, D)
                  for l in range(w.loops)]
            encs[side] = oracle.encode_side(np.stack(xl), w.bits, w.group)
            del xl
            for loop in range(w.loops):
                g = gpu_component(gc, 0, side, loop, bsel, hsel)
                g = {k: (None if v is None else v[:, :, :T]) for k, v in g.items()}
                assert_component_equal(g, encs[side][loop], None,
                                       f"rows {b0}.. side {side} loop {loop}")
        bi, hi = np.ix_(bsel, hsel)
        for loop in range(w.loops):
            kh = oracle.reconstruct(encs[0], loop, w.bits, w.group).reshape(len(bsel), w.heads, T, D)
            vh = oracle.reconstruct(encs[1], loop, w.bits, w.group).reshape(len(bsel), w.heads, T, D)
            ref = oracle.decode_attention(kh, vh, q[loop][bi, hi], [T] * len(bsel),
                                          kc[loop][bi, hi], vc[loop][bi, hi])
            del kh, vh
            got = outs[loop][np.ix_(bsel, hsel)]
            err = float(np.max(np.abs(got - ref)))
            assert err <= attn_tolerance(ref), (b0, loop, err, attn_tolerance(ref))
            units += len(bsel) * w.heads
        del encs
    assert units == w.batch * w.heads * w.loops
