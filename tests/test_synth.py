"""The shared seeded generator: its hash against the published SplitMix64
output function, its distributions, and slice independence."""
import numpy as np
import torch

import residual_bit_kv_b200.synth as synth


def test_splitmix64_known_values():
    # SplitMix64 with state 0: the first outputs of the published generator
    # (state += golden gamma, then the output function).
    outs, state = [], 0
    for _ in range(3):
        state = (state + synth.GAMMA) & synth.MASK64
        outs.append(synth.mix64_py(state))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_tensor_hash_matches_python_form():
    idx = torch.tensor([0, 1, 2, 12345, 2 ** 40 + 7, 2 ** 50 + 3], dtype=torch.int64)
    key = synth.stream_key(3, 5, 1, 2, synth.KIND_N)
    got = synth.hash_t(key, idx).numpy().view(np.uint64)
    want = np.array([synth.hash_py(key, int(i)) for i in idx], dtype=np.uint64)
    np.testing.assert_array_equal(got, want)


def test_normal_and_uniform_moments():
    idx = torch.arange(200000, dtype=torch.int64)
    n = synth.normal_t(synth.stream_key(0, 0, 0, 0, 1), idx)
    assert abs(n.mean().item()) < 0.01 and abs(n.std().item() - 1) < 0.01
    assert torch.all(n * 65536 == torch.round(n * 65536))        # exact multiples of 2^-16
    u = synth.uniform_t(synth.stream_key(0, 0, 0, 0, 2), idx)
    assert 0 < u.min().item() and u.max().item() < 1 and abs(u.mean().item() - 0.5) < 0.01


def test_slices_are_independent_of_the_request():
    w = synth.WORKLOADS["ouro_layer"].replace(batch=3, heads=4, tokens=40)
    full = synth.kv_full(w, 0, synth.SIDE_K, 1, 0, 40)
    part = synth.kv(w, 0, synth.SIDE_K, 1, [2], [1, 3], 17, 33)
    assert torch.equal(part, full[2:3, [1, 3], 17:33])
    cur = synth.current_token(w, 0, synth.SIDE_V, 2)
    assert torch.equal(cur, synth.kv_full(w, 0, synth.SIDE_V, 2, 40, 41)[:, :, 0])


def test_loops_are_correlated_with_the_anchor():
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=256)
    xa = synth.kv_full(w, 0, synth.SIDE_V, 3, 0, 256).float()
    for r, sig in enumerate(w.sigma):
        xr = synth.kv_full(w, 0, synth.SIDE_V, r, 0, 256).float()
        resid = (xr - xa * (xr * xa).sum(-1, keepdim=True) / (xa * xa).sum(-1, keepdim=True))
        assert abs(resid.std().item() - sig) < 0.05 * sig + 0.01


def test_batch_partition_reproduces_the_global_rows():
    """A rank's share of a batch generates exactly those rows of the global
    workload: states, queries, current tokens and ragged lengths."""
    w = synth.WORKLOADS["ouro_layer"].replace(batch=5, heads=2, tokens=24)
    full_k = synth.kv_full(w, 0, synth.SIDE_K, 1, 0, 24)
    full_q = synth.query(w, 0, 2)
    full_c = synth.current_token(w, 0, synth.SIDE_V, 0)
    full_l = synth.seq_lens_ragged(w)
    rows = []
    for r in range(3):
        p = synth.partition(w, r, 3)
        lo = r * 5 // 3
        assert p.batch0 == lo and p.batch == (r + 1) * 5 // 3 - lo
        rows += list(range(lo, lo + p.batch))
        assert torch.equal(synth.kv_full(p, 0, synth.SIDE_K, 1, 0, 24), full_k[lo:lo + p.batch])
        assert torch.equal(synth.query(p, 0, 2), full_q[lo:lo + p.batch])
        assert torch.equal(synth.current_token(p, 0, synth.SIDE_V, 0), full_c[lo:lo + p.batch])
        assert synth.seq_lens_ragged(p) == full_l[lo:lo + p.batch]
    assert rows == list(range(5))
