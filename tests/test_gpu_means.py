"""Fixed means of the residual loops (rq_cache_set_means) through the C ABI vs
the oracle: bit-exact codes, metadata and LS coefficients (per-loop and fused
appends), decode attention within 2e-3 * max|out| on compiled and generic
kernels, and the reconstruction export."""
import numpy as np
import pytest
import torch

import oracle
import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import (SIDES, Workspace, assert_component_equal, attn_tolerance,
                        build_gpu_cache, gpu_component, gpu_decode, mean_rows, oracle_decode,
                        oracle_encode)

pytestmark = pytest.mark.gpu


def _inputs(gc, side, T, bsel, hsel):
    w = gc.w
    return [synth.bits_of(gc.inputs[(0, side, l)][bsel][:, hsel, :T].cpu()).reshape(-1, w.head_dim)
            for l in range(w.loops)]


@pytest.mark.parametrize("policy", ["last", "next", "first", "previous"])
@pytest.mark.parametrize("fused", [False, True])
def test_means_append_bit_exact(cuda_dev, policy, fused):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=200)
    gc = build_gpu_cache(w, policy=policy, fused=fused, means_seed=5, append_chunks=[150, 1, 49])
    bsel, hsel = [0, 1], [0, 1, 2]
    for side in SIDES:
        encs, _ = oracle_encode(w, 0, side, bsel, hsel, 0, 200, policy, _inputs(gc, side, 200, bsel, hsel),
                                means=gc.means)
        for loop in range(w.loops):
            g = gpu_component(gc, 0, side, loop, bsel, hsel)
            g = {k: (None if v is None else v[:, :, :200]) for k, v in g.items()}
            assert_component_equal(g, encs[loop], None, f"means side {side} loop {loop}")


@pytest.mark.parametrize("policy", ["last", "next", "previous"])
def test_means_decode(cuda_dev, policy):
    bits = (2, 2, 2, 4) if policy in ("last", "next") else (4, 2, 2, 2)
    for b, g in ((bits, (32, 32, 32, 32)), ((4, 2, 2, 4), (16, 64, 128, 32))):   # compiled, generic
        w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=300, bits=b, group=g)
        gc = build_gpu_cache(w, policy=policy, means_seed=7)
        ws = Workspace(gc.layout, 300)
        for loop in range(w.loops):
            out, status = gpu_decode(gc, 0, loop, [300, 111], 300, ws)
            assert status == L.RQ_OK
            ref = oracle_decode(w, 0, loop, [0, 1], [0, 1], [300, 111], policy, gc.inputs,
                                means=gc.means)
            err = np.max(np.abs(out - ref))
            assert err <= attn_tolerance(ref), (b, g, loop, err)


def test_means_export(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=64)
    gc = build_gpu_cache(w, policy="next", means_seed=9)
    for side in SIDES:
        encs, _ = oracle_encode(w, 0, side, [0], [0, 1], 0, 64, "next", _inputs(gc, side, 64, [0], [0, 1]),
                                means=gc.means)
        for loop in range(w.loops):
            out = torch.empty(w.batch, w.heads, 64, w.head_dim, dtype=torch.float32, device="cuda")
            L.rq_dequantize(gc.cache, 0, side, loop, 0, 64, out)
            torch.cuda.synchronize()
            ref = oracle.reconstruct(encs, loop, w.bits, w.group, "next",
                                     mean_rows(w, 0, side, [0], [0, 1], 64, gc.means))
            np.testing.assert_allclose(out.cpu().numpy().reshape(-1, w.head_dim), ref,
                                       rtol=2e-6, atol=2e-6 * float(np.abs(ref).max()))
