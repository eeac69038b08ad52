"""The device-side failure path without a GPU fault: a bounded wait that nothing
completes runs out, the error word reports RQ_ERR_TIMEOUT, and the context
keeps working (a decode afterwards still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import residual_bit_kv_b200.librq as L
import residual_bit_kv_b200.synth as synth
from rq_harness import Workspace, attn_tolerance, build_gpu_cache, gpu_decode, oracle_decode

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_dev):
    w = synth.WORKLOADS["tiny"]
    gc = build_gpu_cache(w)
    ws = Workspace(gc.layout, w.tokens)
    t0 = time.perf_counter()
    L.rq_selftest_wait_timeout(ws.buf, ws.bytes, 50)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert L.rq_workspace_error(ws.buf, ws.bytes) == L.RQ_ERR_TIMEOUT
    assert 0.04 <= dt < 5.0, dt
    assert L.rq_workspace_error(ws.buf, ws.bytes) == L.RQ_OK   # read and cleared
    out, status = gpu_decode(gc, 0, 0, [w.tokens], w.tokens, ws)
    assert status == L.RQ_OK
    ref = oracle_decode(w, 0, 0, [0], list(range(w.heads)), [w.tokens])
    assert np.max(np.abs(out - ref)) <= attn_tolerance(ref)
