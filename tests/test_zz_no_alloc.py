"""rq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (the split-K scratch is a fixed array inside librq).

It must give the results of the workspace entry point, on consecutive calls
that reuse the shared scratch, and refuse shapes whose split partials cannot
fit.  Collected last on purpose (file name): it holds the library's static
scratch and must pass both alone and after every other test.
"""
import numpy as np
import pytest
import torch

import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import (Workspace, attn_tolerance, build_gpu_cache, decode_inputs, gpu_decode,
                        oracle_decode)

pytestmark = pytest.mark.gpu


def _noalloc(gc, layer, loop, seq, max_len):
    w = gc.w
    q, kc, vc = decode_inputs(w, layer, loop)
    sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
    out = torch.full((w.batch, w.heads, w.head_dim), float("nan"), dtype=torch.float32,
                     device="cuda")
    L.rq_decode_attention_noalloc(gc.cache, layer, loop, q, sl, max_len, kc, vc, 0.0, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("policy", ["last", "next"])
def test_noalloc_matches_workspace_entry_point(cuda_dev, policy):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=3, heads=4, tokens=700)
    gc = build_gpu_cache(w, policy=policy)
    seq = [700, 333, 0]
    for loop in (0, 2, 3):
        ws_out, status = gpu_decode(gc, 0, loop, seq, 700)
        assert status == L.RQ_OK
        ref = oracle_decode(w, 0, loop, list(range(w.batch)), list(range(w.heads)), seq, policy,
                            gc.inputs)
        for _ in range(2):   # two calls in a row share the static scratch
            got = _noalloc(gc, 0, loop, seq, 700)
            assert np.all(np.isfinite(got))
            # against the oracle, and against the workspace entry point
            assert np.max(np.abs(got - ref)) <= attn_tolerance(ref), (policy, loop)
            assert np.max(np.abs(got - ws_out)) <= attn_tolerance(ws_out), (policy, loop)


def test_noalloc_marks_invalid_rows_nan(cuda_dev):
    """The no-allocation call has no workspace error word for the caller to
    read, so a (batch, head) whose decode is not valid comes back as a NaN row:
    here one unit's value weights pass the accumulator range (the case the
    workspace entry point reports as RQ_ERR_UNSUPPORTED); the other unit
    matches the oracle."""
    import range_case as rc
    bits = rc.inputs()
    lay, cache, keep, q, kc, vc = rc.build(bits)
    sl = torch.full((rc.B,), rc.T, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.zeros(rc.B, rc.H, rc.D, dtype=torch.float32, device="cuda")
        L.rq_decode_attention_noalloc(cache, 0, 0, q, sl, rc.T, kc, vc, 0.0, out)
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(np.isnan(got[0]))
        ref = rc.oracle_out(bits, 1, 0)
        assert np.max(np.abs(got[1, 0] - ref)) <= attn_tolerance(ref)


def _noalloc_fit(bh, D=128):
    """Split partials that fit the no-allocation scratch (8 MiB: error word,
    a counter per row for up to 65535 rows at 256 bytes, then the partials,
    256-aligned)."""
    poff = -(-(256 + 65535 * 4) // 256) * 256
    return ((8 << 20) - poff) // (bh * (D + 2) * 4)


def test_noalloc_fewer_splits_when_partials_do_not_fit(cuda_dev):
    """A shape whose split plan needs more partials than the scratch holds
    runs with fewer, longer splits and still equals the workspace entry point:
    batch 2221 (one head), 32768 past tokens, 2 loops (about 19 GB of packed
    cache, filled from Gaussian rows)."""
    T, D = 32768, 128
    bh = None
    for b in range(2221, 2400):
        lay = L.make_layout(1, 2, b, 1, D, T, (2, 4), (32, 32))
        if L.rq_decode_splits(lay, T) > _noalloc_fit(b):
            bh = b
            break
    assert bh is not None, "no shape in range takes the fewer-splits path on this device"
    nb = L.rq_cache_bytes(lay)
    kb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    vb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    cache = L.rq_cache_bind(lay, kb, vb)
    g = torch.Generator(device="cuda").manual_seed(3)
    step = 2048
    for side in (0, 1):
        for t0 in range(0, T, step):
            a = torch.randn(bh, 1, step, D, generator=g, device="cuda").to(torch.bfloat16)
            L.rq_quantize_anchor(cache, 0, side, a, t0, step)
            r = (a.float() * 0.9 + 0.3 * torch.randn(bh, 1, step, D, generator=g, device="cuda"))
            L.rq_quantize_append_residual(cache, 0, side, 0, r.to(torch.bfloat16), t0, step)
            del a, r
    q, kc, vc = (torch.randn(bh, 1, D, generator=g, device="cuda").to(torch.bfloat16)
                 for _ in range(3))
    sl = torch.full((bh,), T, dtype=torch.int32, device="cuda")
    ws = Workspace(lay, T)
    for loop in (0, 1):
        ref = torch.empty(bh, 1, D, dtype=torch.float32, device="cuda")
        L.rq_decode_attention(cache, 0, loop, q, sl, T, kc, vc, 0.0, ref, ws.buf, ws.bytes)
        assert L.rq_workspace_error(ws.buf, ws.bytes) == L.RQ_OK
        for _ in range(2):
            out = torch.full((bh, 1, D), float("nan"), dtype=torch.float32, device="cuda")
            L.rq_decode_attention_noalloc(cache, 0, loop, q, sl, T, kc, vc, 0.0, out)
            torch.cuda.synchronize()
            r_, o_ = ref.cpu().double().numpy(), out.cpu().double().numpy()
            assert np.all(np.isfinite(o_))
            assert np.max(np.abs(o_ - r_)) <= attn_tolerance(r_), loop
    del kb, vb, cache
    torch.cuda.empty_cache()


def test_noalloc_rejects_shapes_that_do_not_fit(cuda_dev):
    # 65535 (batch, head) rows x 130 floats x 4 bytes exceeds the scratch even
    # with one split: refused on the host, nothing is launched (the cache
    # pointers below are never dereferenced).
    lay = L.make_layout(1, 2, 65535, 1, 128, 64, (2, 4), (32, 32))
    cache = L.rq_cache_bind(lay, 1 << 20, 1 << 30)
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention_noalloc(cache, 0, 0, 256, 256, 64, 256, 256, 0.0, 256)
    assert e.value.status == L.RQ_ERR_WORKSPACE
