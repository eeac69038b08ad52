"""GPU quantise-and-append through the C ABI vs the oracle: packed codes,
fp16 metadata and bf16 LS coefficients must be bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import residual_bit_kv_b200.synth as synth
from rq_harness import (SIDES, assert_component_equal, build_gpu_cache, gpu_component,
                        oracle_encode)

pytestmark = pytest.mark.gpu


def _check_all(gc, layer=0, tokens=None, bsel=None, hsel=None, from_gpu_inputs=True):
    w = gc.w
    T = w.tokens if tokens is None else tokens
    bsel = list(range(w.batch)) if bsel is None else bsel
    hsel = list(range(w.heads)) if hsel is None else hsel
    for side in SIDES:
        xl = None
        if from_gpu_inputs:
            xl = [synth.bits_of(gc.inputs[(layer, side, l)][bsel][:, hsel].cpu()).reshape(-1, w.head_dim)
                  for l in range(w.loops)]
        encs, _ = oracle_encode(w, layer, side, bsel, hsel, 0, T, gc.policy, xl, gc.unit_alpha)
        for loop in range(w.loops):
            g = gpu_component(gc, layer, side, loop, bsel, hsel)
            gsel = {k: (None if v is None else v[:, :, :T]) for k, v in g.items()}
            assert_component_equal(gsel, encs[loop], None, f"side {side} loop {loop}")


def test_generator_identical_on_cuda(cuda_dev):
    """The shared generator draws the same bf16 values on the GPU and the host."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=50)
    for side in SIDES:
        for loop in range(w.loops):
            a = synth.kv_full(w, 0, side, loop, 0, 50, device="cuda").cpu()
            b = synth.kv_full(w, 0, side, loop, 0, 50, device="cpu")
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(synth.query(w, 0, 1, "cuda").cpu().view(torch.int16),
                       synth.query(w, 0, 1, "cpu").view(torch.int16))


def test_tiny_reference_bit_exact(cuda_dev):
    """Tiny reference workload (2 loops, D=64, 256 tokens): every stored bit."""
    gc = build_gpu_cache(synth.WORKLOADS["tiny"])
    _check_all(gc, from_gpu_inputs=False)


@pytest.mark.parametrize("bits,group,policy", [
    ((2, 2, 2, 4), (32, 32, 32, 32), "last"),
    ((4, 2, 2, 4), (32, 32, 32, 32), "last"),
    ((2, 2, 2, 4), (16, 16, 16, 32), "last"),
    ((2, 2, 4, 4), (64, 64, 16, 16), "last"),
    ((2, 2, 2, 4), (128, 32, 64, 128), "next"),
    ((2, 4, 2, 4), (32, 32, 32, 64), "next"),
    ((4, 2, 2, 2), (32, 32, 32, 32), "first"),
    ((4, 2, 4, 2), (32, 16, 64, 128), "previous"),
])
def test_ragged_shapes_bit_exact(cuda_dev, bits, group, policy):
    """Several warps, a ragged row tail and every bit-width / group size."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=203, bits=bits, group=group)
    gc = build_gpu_cache(w, policy=policy)
    _check_all(gc)


def test_head_dim_64_chained_bit_exact(cuda_dev):
    w = synth.WORKLOADS["huginn_deep"].replace(batch=1, heads=3, tokens=77, head_dim=64, loops=5,
                                               bits=(2, 2, 4, 2, 4), group=(32, 16, 64, 64, 32),
                                               sigma=(0.4, 0.3, 0.2, 0.1))
    gc = build_gpu_cache(w, policy="next")
    _check_all(gc)


def test_appends_match_prefill(cuda_dev):
    """Prefill followed by single-token appends at t0 = T, T+1, ... stores the
    same bits as the oracle's whole-sequence encoding (rows are independent)."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=133)
    gc = build_gpu_cache(w, append_chunks=[128, 1, 1, 3])
    _check_all(gc)


def test_edge_rows(cuda_dev):
    """Zero rows (zero anchor -> alpha 0, constant groups -> codes 0), a row
    equal to a power-of-two multiple of the anchor, and huge/small magnitudes."""
    import residual_bit_kv_b200.librq as L
    from rq_harness import layout_of
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=1, tokens=8)
    lay = layout_of(w, max_tokens=8)
    nb = L.rq_cache_bytes(lay)
    kb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    vb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    cache = L.rq_cache_bind(lay, kb, vb)
    g = torch.Generator().manual_seed(0)
    anchor = torch.randn(1, 1, 8, 128, generator=g)
    anchor[0, 0, 0] = 0.0                       # zero anchor row
    anchor[0, 0, 1] = 3.0                       # constant row
    anchor[0, 0, 5] *= 1e3
    anchor[0, 0, 6] *= 1e-3
    xs = {3: anchor.to(torch.bfloat16)}
    for r in range(3):
        x = anchor * 0.9 + 0.2 * torch.randn(1, 1, 8, 128, generator=g)
        x[0, 0, 2] = anchor[0, 0, 2] * 2.0      # exact multiple of the anchor input
        x[0, 0, 3] = 0.0
        xs[r] = x.to(torch.bfloat16)
    for side in (0, 1):
        L.rq_quantize_anchor(cache, 0, side, xs[3].cuda(), 0, 8)
        for r in (2, 1, 0):
            L.rq_quantize_append_residual(cache, 0, side, r, xs[r].cuda(), 0, 8)
    torch.cuda.synchronize()
    x = np.stack([synth.bits_of(xs[l]).reshape(-1, 128) for l in range(4)])
    encs = oracle.encode_side(x, w.bits, w.group)
    from rq_harness import GpuCache
    gc = GpuCache(w, "last", lay, cache, kb, vb, {})
    for side in (0, 1):
        for loop in range(4):
            gcomp = gpu_component(gc, 0, side, loop)
            gsel = {k: (None if v is None else v[:, :, :8]) for k, v in gcomp.items()}
            assert_component_equal(gsel, encs[loop], None, f"edge loop {loop}")
    assert encs[0]["alpha"][0] == 0                       # zero anchor -> alpha 0


def test_dequantize_matches_oracle(cuda_dev):
    import residual_bit_kv_b200.librq as L
    for policy in ("last", "next"):
        w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=150)
        gc = build_gpu_cache(w, policy=policy)
        for side in SIDES:
            encs, _ = oracle_encode(w, 0, side, [0, 1], [0, 1], 0, 150, policy)
            for loop in range(w.loops):
                out = torch.empty(2, 2, 100, 128, dtype=torch.float32, device="cuda")
                L.rq_dequantize(gc.cache, 0, side, loop, 25, 100, out)
                torch.cuda.synchronize()
                ref = oracle.reconstruct(encs, loop, w.bits, w.group, policy).reshape(2, 2, 150, 128)
                ref = ref[:, :, 25:125]
                err = np.max(np.abs(out.cpu().numpy() - ref))
                assert err <= 2e-6 * np.max(np.abs(ref)) + 1e-7, (policy, side, loop, err)


# ---- every loop of a layer, both sides, in one launch (rq_quantize_append_loops)

@pytest.mark.parametrize("bits,group,policy", [
    ((2, 2, 2, 4), (32, 32, 32, 32), "last"),
    ((4, 2, 2, 4), (32, 32, 32, 32), "last"),
    ((2, 2, 2, 4), (16, 16, 16, 32), "last"),
    ((2, 2, 4, 4), (64, 64, 16, 16), "next"),
    ((2, 2, 2, 4), (128, 32, 64, 128), "next"),
    ((4, 2, 2, 2), (32, 32, 32, 32), "first"),
    ((4, 2, 4, 2), (32, 16, 64, 128), "previous"),
])
def test_fused_loops_bit_exact(cuda_dev, bits, group, policy):
    """One launch per chunk stores the bits of the per-loop path: codes,
    metadata and LS coefficients of every loop against the oracle."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=203, bits=bits, group=group)
    gc = build_gpu_cache(w, policy=policy, fused=True)
    _check_all(gc)


def test_fused_loops_head_dim_64_deep_chain(cuda_dev):
    w = synth.WORKLOADS["huginn_deep"].replace(batch=1, heads=3, tokens=77, head_dim=64, loops=5,
                                               bits=(2, 2, 4, 2, 4), group=(32, 16, 64, 64, 32),
                                               sigma=(0.4, 0.3, 0.2, 0.1))
    gc = build_gpu_cache(w, policy="next", fused=True)
    _check_all(gc)


def test_fused_single_token_appends(cuda_dev):
    """Prefill then single-token appends of every loop (the decode step's
    append) through the fused entry point."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=133)
    gc = build_gpu_cache(w, append_chunks=[128, 1, 1, 3], fused=True)
    _check_all(gc)


def test_fused_one_side_leaves_the_other(cuda_dev):
    """xv = NULL appends K only: K matches the oracle over the longer sequence
    and the V cache bytes are untouched."""
    import residual_bit_kv_b200.librq as L
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=64)
    gc = build_gpu_cache(w, fused=True, max_tokens=128)
    before = gc.vbuf.clone()
    xk = torch.stack([synth.kv_full(w, 0, synth.SIDE_K, l, 64, 66, device="cuda")
                      for l in range(w.loops)]).contiguous()
    L.rq_quantize_append_loops(gc.cache, 0, xk, None, 64, 2)
    torch.cuda.synchronize()
    assert torch.equal(before, gc.vbuf)
    w66 = w.replace(tokens=66)
    encs, _ = oracle_encode(w66, 0, synth.SIDE_K, [0], [0, 1], 0, 66, "last")
    for loop in range(w.loops):
        g = gpu_component(gc, 0, synth.SIDE_K, loop)
        g = {k: (None if v is None else v[:, :, :66]) for k, v in g.items()}
        assert_component_equal(g, encs[loop], None, f"K loop {loop}")


@pytest.mark.parametrize("policy,fused", [("last", False), ("next", True), ("first", True),
                                          ("previous", False)])
def test_unit_alpha_bit_exact(cuda_dev, policy, fused):
    """alpha = 1 (RQ_FLAG_UNIT_ALPHA): plain differences against the reference,
    every alpha stored as bf16(1.0), both append paths."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=97)
    gc = build_gpu_cache(w, policy=policy, fused=fused, unit_alpha=True)
    _check_all(gc)
    a = oracle.anchor_loop(w.loops, policy)
    for loop in range(w.loops):
        if loop != a:
            al = gpu_component(gc, 0, 0, loop)["alpha"][:, :, :w.tokens]
            assert np.all(al == 0x3F80)


def test_first_loop_deep_head_dim_64_bit_exact(cuda_dev):
    w = synth.WORKLOADS["huginn_deep"].replace(batch=1, heads=3, tokens=77, head_dim=64, loops=5,
                                               bits=(4, 2, 2, 4, 2), group=(32, 16, 64, 64, 32),
                                               sigma=(0.4, 0.3, 0.2, 0.1))
    for policy in ("first", "previous"):
        for fused in (False, True):
            gc = build_gpu_cache(w, policy=policy, fused=fused)
            _check_all(gc)


# ---- degenerate rows and extreme magnitudes, through the C ABI on given rows

def _encode_given_rows(x_loops, bits, group, policy="last"):
    """x_loops: uint16 numpy [L, N, D] bf16 bits.  Quantises them through the
    C ABI (per-loop and fused paths) as batch 1, N heads, 1 token, and returns
    (gpu components of both paths, oracle encodings)."""
    import residual_bit_kv_b200.librq as L
    from rq_harness import policy_code
    Lp, N, D = x_loops.shape
    lay = L.make_layout(1, Lp, 1, N, D, 64, bits, group, policy_code(policy))
    nb = L.rq_cache_bytes(lay)
    out = []
    for fused in (False, True):
        kb = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        vb = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        cache = L.rq_cache_bind(lay, kb, vb)
        xs = torch.from_numpy(x_loops.astype(np.int16)).view(torch.bfloat16).cuda()
        if fused:
            L.rq_quantize_append_loops(cache, 0, xs.contiguous(), None, 0, 1)
        else:
            a = oracle.anchor_loop(Lp, policy)
            for loop in [a] + oracle.encode_order(Lp, policy):
                x = xs[loop].contiguous()
                if loop == a:
                    L.rq_quantize_anchor(cache, 0, 0, x, 0, 1)
                else:
                    L.rq_quantize_append_residual(cache, 0, 0, loop, x, 0, 1)
        torch.cuda.synchronize()
        w = synth.WORKLOADS["tiny"].replace(loops=Lp, batch=1, heads=N, head_dim=D, tokens=1,
                                           bits=tuple(bits), group=tuple(group))
        from rq_harness import GpuCache
        gc = GpuCache(w, policy, lay, cache, kb, vb, {})
        out.append([{k: (None if v is None else v[:, :, :1]) for k, v in
                     gpu_component(gc, 0, 0, loop).items()} for loop in range(Lp)])
    return out, oracle.encode_side(x_loops, bits, group, policy)


def _bf16_bits(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def test_degenerate_rows_bit_exact(cuda_dev):
    """Zero rows, constant rows (every group range 0: s~ = 0, codes 0),
    a single non-zero channel, and loops equal to the anchor (zero residual)."""
    D = 128
    rows = np.zeros((6, D), np.float32)
    rows[1] = 3.25                                   # constant row
    rows[2, 17] = -7.0                               # one non-zero channel
    rows[3] = np.linspace(-1, 1, D)
    rows[4] = -0.0                                   # negative zero
    rows[5, ::2] = 1e-30                             # subnormal after rotation
    anchor = _bf16_bits(rows)
    loops = np.stack([anchor, _bf16_bits(rows * 0.5), _bf16_bits(np.zeros_like(rows)), anchor])
    for policy in ("last", "next"):
        (per_loop, fused), encs = _encode_given_rows(loops, (2, 2, 2, 4), (32, 16, 64, 32), policy)
        for got in (per_loop, fused):
            for r in range(4):
                assert_component_equal(got[r], encs[r], None, f"{policy} loop {r}")


def test_extreme_magnitudes_bit_exact(cuda_dev):
    """Large magnitudes with tiny ranges (the fp16 offset's rounding exceeds
    a quantisation step, so the clamps decide codes), spikes near the fp16
    limit after rotation, and very small values: bit-exact on both sides.
    Inputs stay where the fp16 scale and offset are finite; beyond that the
    method produces NaN metadata, whose bit pattern the pages do not fix."""
    D = 64
    rng = np.random.default_rng(3)
    rows = rng.standard_normal((8, D)).astype(np.float32)
    rows[0] *= 2000.0
    rows[1] = 5e3 + 1e-2 * rows[1]                   # range far below the offset's ulp
    rows[2, :5] = 7999.0
    rows[3] *= 1e-6
    rows[4, 0] = 8000.0
    rows[5] = 1000.0 + np.arange(D, dtype=np.float32)
    rows[6, 10] = -8000.0
    anchor = _bf16_bits(rows)
    loops = np.stack([_bf16_bits(rows[::-1].copy()), anchor])
    for bits in ((2, 4), (4, 2)):
        (per_loop, fused), encs = _encode_given_rows(loops, bits, (32, 64), "last")
        for r in range(2):
            m = encs[r]["meta"]
            assert not np.any(((m & 0x7C00) == 0x7C00) & ((m & 0x3FF) != 0))
            assert not np.any((((m >> 16) & 0x7C00) == 0x7C00) & (((m >> 16) & 0x3FF) != 0))
        for got in (per_loop, fused):
            for r in range(2):
                assert_component_equal(got[r], encs[r], None, f"bits {bits} loop {r}")


def test_maximum_loop_count_chain(cuda_dev):
    """RQ_MAX_LOOPS = 32 loops under the Next-loop chain (loop 0 is rebuilt from
    32 components): every code bit-exact, both append paths."""
    import residual_bit_kv_b200.librq as L
    bits = tuple([2] * 31 + [4])
    group = tuple([32] * 32)
    w = synth.WORKLOADS["huginn_deep"].replace(loops=32, batch=1, heads=2, tokens=40, head_dim=64,
                                               bits=bits, group=group,
                                               sigma=tuple(np.linspace(0.4, 0.1, 31)))
    assert w.loops == L.RQ_MAX_LOOPS
    for fused in (False, True):
        gc = build_gpu_cache(w, policy="next", fused=fused)
        _check_all(gc)
