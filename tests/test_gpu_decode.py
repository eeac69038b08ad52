"""GPU decode attention through the C ABI vs the oracle's fp64 attention over
its own reconstruction: max |err| <= 2e-3 * max |out|."""
import numpy as np
import pytest
import torch

import oracle
import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import (Workspace, attn_tolerance, build_gpu_cache, decode_inputs, gpu_decode,
                        oracle_decode)

pytestmark = pytest.mark.gpu


def _check_decode(gc, seq_lens, max_seq_len, loops=None, layer=0, bsel=None, hsel=None):
    w = gc.w
    loops = range(w.loops) if loops is None else loops
    bsel = list(range(w.batch)) if bsel is None else bsel
    hsel = list(range(w.heads)) if hsel is None else hsel
    ws = Workspace(gc.layout, max_seq_len)
    for loop in loops:
        out, status = gpu_decode(gc, layer, loop, seq_lens, max_seq_len, ws)
        assert status == L.RQ_OK
        ref = oracle_decode(w, layer, loop, bsel, hsel, seq_lens, gc.policy, gc.inputs or None,
                            unit_alpha=gc.unit_alpha)
        got = out[np.ix_(bsel, hsel)]
        err = np.max(np.abs(got - ref))
        assert err <= attn_tolerance(ref), (loop, err, attn_tolerance(ref))


def test_tiny_reference_decode(cuda_dev):
    w = synth.WORKLOADS["tiny"]
    gc = build_gpu_cache(w)
    _check_decode(gc, [256], 256)


@pytest.mark.parametrize("policy", ["last", "next", "first", "previous"])
def test_ragged_lengths(cuda_dev, policy):
    """Ragged past lengths (0, a partial chunk, several chunks, full) in one batch."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=4, heads=3, tokens=777)
    gc = build_gpu_cache(w, policy=policy)
    _check_decode(gc, [777, 0, 63, 400], 777)


def test_mixed_precision_and_groups(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=500, bits=(4, 2, 2, 4),
                                              group=(16, 64, 128, 32))
    gc = build_gpu_cache(w)
    _check_decode(gc, [500, 321], 500)


def test_deep_chain_head_dim_64(cuda_dev):
    w = synth.WORKLOADS["huginn_deep"].replace(batch=2, heads=2, tokens=300, head_dim=64)
    for policy in ("last", "next", "first", "previous"):
        gc = build_gpu_cache(w, policy=policy)
        _check_decode(gc, [300, 129], 300, loops=[0, 3, 6, 7])


@pytest.mark.parametrize("policy", ["last", "previous"])
def test_unit_alpha_decode(cuda_dev, policy):
    """alpha = 1 (no LS scaling, [RQ Table 3]): plain inter-loop differences."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=3, tokens=300,
                                              bits=(4, 2, 2, 2) if policy == "previous"
                                              else (2, 2, 2, 4))
    gc = build_gpu_cache(w, policy=policy, unit_alpha=True)
    _check_decode(gc, [300, 77], 300)


def test_no_past_tokens_returns_current_value(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=64)
    gc = build_gpu_cache(w)
    for max_len in (0, 64):
        out, status = gpu_decode(gc, 0, 1, [0, 0], max_len)
        assert status == L.RQ_OK
        _, _, vc = decode_inputs(w, 0, 1)
        np.testing.assert_array_equal(out, vc.float().cpu().numpy().astype(np.float64))


def test_seq_len_over_bound_is_flagged_and_clamped(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=200)
    gc = build_gpu_cache(w)
    out, status = gpu_decode(gc, 0, 0, [150, 999], 150)
    assert status == L.RQ_ERR_CAPACITY
    ref = oracle_decode(w, 0, 0, [0, 1], [0, 1], [150, 150], "last", gc.inputs)
    assert np.max(np.abs(out - ref)) <= attn_tolerance(ref)
    # the error word is cleared by reading it
    out2, status2 = gpu_decode(gc, 0, 0, [150, 150], 150)
    assert status2 == L.RQ_OK


def test_softmax_scale_argument(cuda_dev):
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=100)
    gc = build_gpu_cache(w)
    out, _ = gpu_decode(gc, 0, 2, [100], 100, scale=0.05)
    ref = oracle_decode(w, 0, 2, [0], [0, 1], [100], "last", gc.inputs, scale=0.05)
    assert np.max(np.abs(out - ref)) <= attn_tolerance(ref)


def test_workspace_reuse_across_calls(cuda_dev):
    """Self-resetting split counters: many calls on one workspace stay exact."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=640)
    gc = build_gpu_cache(w)
    ws = Workspace(gc.layout, 640)
    first, _ = gpu_decode(gc, 0, 1, [640, 333], 640, ws)
    for _ in range(5):
        again, st = gpu_decode(gc, 0, 1, [640, 333], 640, ws)
        assert st == L.RQ_OK
        np.testing.assert_array_equal(again, first)


def test_bf16_decode_matches_oracle(cuda_dev):
    """The uncompressed baseline kernel on the same engine."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=3, heads=2, tokens=450)
    T = w.tokens
    k = synth.kv_full(w, 0, 0, 1, 0, T, device="cuda")
    v = synth.kv_full(w, 0, 1, 1, 0, T, device="cuda")
    q, kc, vc = decode_inputs(w, 0, 1)
    seq = [450, 1, 190]
    sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
    nb = L.rq_decode_bf16_workspace_bytes(3, 2, 128, T)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    out = torch.empty(3, 2, 128, dtype=torch.float32, device="cuda")
    L.rq_decode_attention_bf16(3, 2, 128, q, k, v, T, sl, T, kc, vc, 0.0, out, ws, nb)
    torch.cuda.synchronize()
    kf = k.double().cpu().numpy()
    vf = v.double().cpu().numpy()
    ref = oracle.decode_attention(kf, vf, synth.bits_of(q), seq, synth.bits_of(kc), synth.bits_of(vc))
    got = out.cpu().numpy()
    assert np.max(np.abs(got - ref)) <= attn_tolerance(ref)


def test_maximum_loop_count_chain_decode(cuda_dev):
    """32 loops under the Next-loop chain: loop 0 reads 32 components (the
    layout-generic decode kernel); every loop within tolerance."""
    bits = tuple([2] * 31 + [4])
    w = synth.WORKLOADS["huginn_deep"].replace(loops=32, batch=1, heads=2, tokens=200, head_dim=64,
                                               bits=bits, group=tuple([32] * 32),
                                               sigma=tuple(np.linspace(0.4, 0.1, 31)))
    gc = build_gpu_cache(w, policy="next")
    _check_decode(gc, [200], 200, loops=[0, 1, 15, 30, 31])


@pytest.mark.parametrize("T", [1, 63, 64, 65, 777, 4096, 16384, 65536])
@pytest.mark.parametrize("batch,heads", [(1, 1), (2, 3), (16, 16), (64, 40)])
def test_split_plan_invariants(cuda_dev, T, batch, heads):
    """The split count of a decode call: at least one, no more than the
    workspace holds (one per 64-token chunk), and never an empty split."""
    lay = L.make_layout(1, 4, batch, heads, 128, T, (2, 2, 2, 4), (32,) * 4)
    s = L.rq_decode_splits(lay, T)
    chunks = (T + 63) // 64
    assert 1 <= s <= max(1, chunks)
    cps = -(-chunks // s)
    assert -(-chunks // cps) == s


def test_value_range_limit_gives_nan_rows_and_a_flag(cuda_dev):
    """A unit whose value weights p * alpha * s~ reach 2^36 (the limit of the
    fast kernel's scaled accumulators) is reported (RQ_ERR_UNSUPPORTED) and its
    output row is NaN; the other unit of the same call is exact to the oracle's
    tolerance, and the anchor loop (alpha = 1) of the same cache is fine."""
    import range_case as rc
    bits = rc.inputs()
    lay, cache, keep, q, kc, vc = rc.build(bits)
    ws = Workspace(lay, rc.T)
    sl = torch.full((rc.B,), rc.T, dtype=torch.int32, device="cuda")
    for loop, bad in ((0, True), (1, False)):
        out = torch.zeros(rc.B, rc.H, rc.D, dtype=torch.float32, device="cuda")
        L.rq_decode_attention(cache, 0, loop, q, sl, rc.T, kc, vc, 0.0, out, ws.buf, ws.bytes)
        status = L.rq_workspace_error(ws.buf, ws.bytes)
        got = out.cpu().numpy().astype(np.float64)
        assert status == (L.RQ_ERR_UNSUPPORTED if bad else L.RQ_OK), loop
        assert np.all(np.isnan(got[0])) == bad and np.all(np.isfinite(got[0])) != bad
        for b in ([1] if bad else [0, 1]):
            ref = rc.oracle_out(bits, b, loop)
            assert np.max(np.abs(got[b, 0] - ref)) <= attn_tolerance(ref), (loop, b)
    assert np.all(np.isfinite(rc.oracle_out(bits, 0, 0)))   # the method itself is fine there
