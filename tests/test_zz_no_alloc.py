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
from rq_harness import attn_tolerance, build_gpu_cache, decode_inputs, gpu_decode

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
        ref, status = gpu_decode(gc, 0, loop, seq, 700)
        assert status == L.RQ_OK
        for _ in range(2):   # two calls in a row share the static scratch
            got = _noalloc(gc, 0, loop, seq, 700)
            assert np.all(np.isfinite(got))
            assert np.max(np.abs(got - ref)) <= attn_tolerance(ref), (policy, loop)


def test_noalloc_rejects_shapes_that_do_not_fit(cuda_dev):
    # 65535 (batch, head) rows x 130 floats x 4 bytes exceeds the scratch even
    # with one split: refused on the host, nothing is launched (the cache
    # pointers below are never dereferenced).
    lay = L.make_layout(1, 2, 65535, 1, 128, 64, (2, 4), (32, 32))
    cache = L.rq_cache_bind(lay, 1 << 20, 1 << 30)
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention_noalloc(cache, 0, 0, 256, 256, 64, 256, 256, 0.0, 256)
    assert e.value.status == L.RQ_ERR_WORKSPACE
