"""Pins of the oracle's dense-rotation path [RQ §3.3, App. G.1, App. G.2]
(binary16 rotation matrices, binary16 inputs, fp32 accumulation in an order
the pages leave open) against things other than itself: numpy's binary16
rounding, signed permutations (exactly orthogonal, not symmetric), the
Sylvester-Hadamard path at head_dim 64 (where 1/sqrt(D) = 1/8 is exact in
binary16), brute force over the boxes of the interval encoder, and the
rotated-domain attention identity."""
import numpy as np
import pytest
import scipy.linalg

import residual_bit_kv_b200.synth as synth


def _bf16_bits(a):
    a = np.ascontiguousarray(a, np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)     # exact for bf16-valued input


def _signed_perm(rng, D):
    perm = rng.permutation(D)
    sign = rng.choice([-1.0, 1.0], D)
    u = np.zeros((D, D), np.float32)
    u[np.arange(D), perm] = sign
    return u.astype(np.float16).view(np.uint16), perm, sign


def _hadamard_f16(D):
    return (scipy.linalg.hadamard(D) / np.sqrt(D)).astype(np.float16).view(np.uint16)


def test_dense_rotation_orientation_and_fp16_inputs(oracle_mod):
    """z_i = sign_i * fp16(x_perm(i)) exactly for a signed permutation: pins
    which index of U is the output channel, and the rounding of the bf16
    inputs to binary16 (against numpy), including binary16 subnormals."""
    rng = np.random.default_rng(1)
    D = 128
    u, perm, sign = _signed_perm(rng, D)
    xv = np.concatenate([rng.standard_normal(D // 2) * 3.0,
                         rng.standard_normal(D // 2) * 3e-6]).astype(np.float32)
    x = synth.f32_to_bf16_bits_np(xv) if hasattr(synth, "f32_to_bf16_bits_np") else \
        np.array([oracle_mod.f32_to_bf16_bits(float(v)) for v in xv], np.uint16)
    xb = (x.astype(np.uint32) << 16).view(np.float32)
    z, bound = oracle_mod.rotate_dense(u, x[None])
    want = sign * xb[perm].astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(z[0], want)
    assert np.any(xb[perm].astype(np.float16).astype(np.float32) != xb[perm])   # rounding happened
    assert np.all(bound[0] == 0.0)          # one term per output: nothing is rounded


def test_dense_bound_covers_fp32_orders(oracle_mod):
    """Sequential, reversed and pairwise fp32 sums of the exact products all
    land within the returned bound of the fp64 sum."""
    rng = np.random.default_rng(2)
    D = 128
    u = (rng.standard_normal((D, D)) / np.sqrt(D)).astype(np.float16)
    x = np.array([oracle_mod.f32_to_bf16_bits(float(v)) for v in rng.standard_normal(D) * 2],
                 np.uint16)
    z, bound = oracle_mod.rotate_dense(u.view(np.uint16), x[None])
    xh = ((x.astype(np.uint32) << 16).view(np.float32)).astype(np.float16).astype(np.float32)
    prods = u.astype(np.float32) * xh[None, :]                 # exact in fp32
    seq = np.zeros(D, np.float32)
    rev = np.zeros(D, np.float32)
    for j in range(D):
        seq = (seq + prods[:, j]).astype(np.float32)
        rev = (rev + prods[:, D - 1 - j]).astype(np.float32)
    pair = prods.copy()
    while pair.shape[1] > 1:
        pair = (pair[:, 0::2] + pair[:, 1::2]).astype(np.float32)
    for got in (seq, rev, pair[:, 0]):
        assert np.all(np.abs(got.astype(np.float64) - z[0]) <= bound[0])
    assert np.any(seq.astype(np.float64) != z[0])             # the bound is doing work


def _narrow_range_rows(rng, n, D):
    """bf16 rows with |x| in [1/8, 8): 8-bit significands over a 2^6 range, so
    every partial sum of a 64-point Hadamard transform needs at most 20 bits
    and is exact in fp32 in any order."""
    mag = np.exp2(rng.uniform(-3, 3, (n, D)))
    v = (mag * rng.choice([-1.0, 1.0], (n, D))).astype(np.float32)
    return _bf16_bits(v) & np.uint16(0xFFFF)   # truncation keeps |x| inside the range


def test_dense_exact_sums_have_zero_bound(oracle_mod):
    """U = P H_128 / 8 (signed row permutation of a Hadamard matrix, entries
    +-1/8 exact in binary16) on bf16 rows with |x| in [1/8, 8): every product
    is a multiple of 2^-13 and their magnitudes sum below 2^11, so every order
    of fp32 accumulation is exact.  The oracle returns a zero bound and z
    equals the sequential, reversed and pairwise fp32 sums bit for bit; a
    random orthogonal U on the same rows gets a positive bound."""
    rng = np.random.default_rng(7)
    D = 128
    perm = rng.permutation(D)
    sign = rng.choice([-1.0, 1.0], D)
    u = (sign[:, None] * scipy.linalg.hadamard(D)[perm] / 8).astype(np.float16)
    x = _narrow_range_rows(rng, 4, D)
    z, bound = oracle_mod.rotate_dense(u.view(np.uint16), x)
    assert np.all(bound == 0.0)
    lo, hi, mid = oracle_mod.f32_box(z, bound)          # boxes of one point
    assert np.array_equal(lo, mid) and np.array_equal(hi, mid)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    prods = u.astype(np.float32)[None, :, :] * xf[:, None, :]
    seq = np.zeros((4, D), np.float32)
    rev = np.zeros((4, D), np.float32)
    for j in range(D):
        seq = (seq + prods[:, :, j]).astype(np.float32)
        rev = (rev + prods[:, :, D - 1 - j]).astype(np.float32)
    np.testing.assert_array_equal(seq.astype(np.float64), z)
    np.testing.assert_array_equal(rev.astype(np.float64), z)
    q, _ = np.linalg.qr(rng.standard_normal((D, D)))
    _, b2 = oracle_mod.rotate_dense(q.astype(np.float16).view(np.uint16), x)
    assert np.all(b2 > 0.0)


@pytest.mark.parametrize("policy", ["last", "next"])
@pytest.mark.parametrize("meta16,means", [(False, False), (True, False), (False, True),
                                          (True, True)])
def test_dense_hadamard_reproduces_fwht_path_bit_for_bit(oracle_mod, policy, meta16, means):
    """U = H_64 / 8 (exact in binary16), on rows whose Hadamard sums are exact
    in any order: the dense encoder's codes, metadata and LS coefficients equal
    the Sylvester-Hadamard (FWHT) encoder's bit for bit, with either metadata
    form and with or without fixed means, and every decision is certified."""
    rng = np.random.default_rng(3)
    D, L, H, T = 64, 4, 2, 40
    xa = _narrow_range_rows(rng, H * T, D)
    xaf = (xa.astype(np.uint32) << 16).view(np.float32)
    # loops as scaled, perturbed copies of the anchor (|x| stays in [2^-4, 16):
    # the 64-point sums still need at most 21 bits)
    x = np.stack([_bf16_bits(((xaf * a * np.exp2(rng.uniform(-0.3, 0.3, (H * T, D))))
                              .astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32))
                  for a in (0.8, 1.1, 0.9)] + [xa])
    u = np.stack([_hadamard_f16(D)] * H)
    bits, group = (2, 2, 2, 4), (32, 32, 32, 32)
    mu = None
    if means:   # fixed means on a 1/64 grid: their subtraction is exact as well
        mu = (rng.integers(-64, 64, (L, H * T, D)) / 64).astype(np.float32)
    want = oracle_mod.encode_side(x, bits, group, policy, meta16=meta16, mu=mu)
    got = oracle_mod.encode_side_dense(x, u, H, T, bits, group, policy, meta16=meta16, mu=mu)
    for l in range(L):
        np.testing.assert_array_equal(got[l]["codes"], want[l]["codes"])
        np.testing.assert_array_equal(got[l]["meta"], want[l]["meta"])
        if want[l]["alpha"] is not None:
            np.testing.assert_array_equal(got[l]["alpha"], want[l]["alpha"])
    # every sum here is exact in any order: every decision is certified
    for l in range(L):
        assert got[l]["clean"].all(), l
    if meta16:   # 16-bit metadata needs exact sums
        q, _ = np.linalg.qr(rng.standard_normal((D, D)))
        uq = np.stack([q.astype(np.float16).view(np.uint16)] * H)
        with pytest.raises(ValueError):
            oracle_mod.encode_side_dense(x, uq, H, T, bits, group, policy, meta16=True)


def _box_samples(rng, lo, hi, k):
    """k fp32 rows inside [lo, hi]: both corners and uniform draws."""
    out = [lo, hi]
    for _ in range(k):
        t = rng.random(lo.shape)
        out.append(np.clip((lo + t * (hi.astype(np.float64) - lo)).astype(np.float32), lo, hi))
    return out


def test_quantize_box_flags_are_sound(oracle_mod):
    """Brute force: every decision flagged as determined is the same for 60
    rows drawn inside the box (corners included); a box that straddles a
    code boundary is not flagged."""
    rng = np.random.default_rng(4)
    D, bits, group = 64, 2, 32
    mid = rng.standard_normal((8, D)).astype(np.float32)
    w = np.abs(mid) * np.exp2(rng.uniform(-20, -8, (8, 1))) + 1e-7   # narrow to wide boxes
    lo = np.nextafter((mid - w).astype(np.float32), np.float32(-np.inf))
    hi = np.nextafter((mid + w).astype(np.float32), np.float32(np.inf))
    codes, meta, _, mok, cok = oracle_mod.quantize_box(lo, hi, mid, bits, group)
    assert cok.any() and not cok.all()
    for r in range(mid.shape[0]):
        for z in _box_samples(rng, lo[r], hi[r], 60):
            words, m, _ = oracle_mod.quantize(z, bits, group)
            c_s = oracle_mod.unpack_codes(words, bits, D)
            c_m = oracle_mod.unpack_codes(codes[r], bits, D)
            assert np.all(c_s[cok[r]] == c_m[cok[r]])
            assert np.all(m[mok[r]] == meta[r][mok[r]])
    # a channel exactly on a rounding boundary with a box around it
    z = np.zeros(D, np.float32)
    z[0], z[1] = 0.0, 3.0                  # s = 1, offset 0, levels 0..3
    z[2] = 1.5                             # the tie between codes 1 and 2
    z[32], z[33] = 0.0, 3.0
    lo = z.copy(); hi = z.copy()
    lo[2] = np.nextafter(np.float32(1.5), np.float32(0))
    hi[2] = np.nextafter(np.float32(1.5), np.float32(9))
    _, _, _, mok, cok = oracle_mod.quantize_box(lo[None], hi[None], z[None], bits, group)
    assert mok.all() and not cok[0, 2] and cok[0, [0, 1, 3, 32, 33]].all()


def test_residual_box_flags_are_sound(oracle_mod):
    """Brute force over the residual encoder: for rows drawn inside the box,
    the flagged LS coefficient, metadata and codes never change."""
    rng = np.random.default_rng(5)
    D, bits, group = 128, 2, 32
    for trial in range(6):
        ref = rng.standard_normal(D).astype(np.float32)
        mid = (0.9 * ref + 0.3 * rng.standard_normal(D)).astype(np.float32)
        w = (np.abs(mid) * 10 ** rng.uniform(-6, -3)).astype(np.float32)
        lo = np.nextafter((mid - w).astype(np.float32), np.float32(-np.inf))
        hi = np.nextafter((mid + w).astype(np.float32), np.float32(np.inf))
        words = np.zeros(D * bits // 32, np.uint32)
        meta = np.zeros(D // group, np.uint32)
        alpha = np.zeros(1, np.uint16)
        zhat = np.zeros(D, np.float32)
        aok = np.zeros(1, np.uint8)
        mok = np.zeros(D // group, np.uint8)
        cok = np.zeros(D, np.uint8)
        P = oracle_mod._ptr
        oracle_mod.lib().rqo_encode_residual_box(P(lo), P(hi), P(mid), P(ref), None, D, bits,
                                                 group, 0, P(words), P(meta), P(alpha),
                                                 P(zhat), P(aok), P(mok), P(cok))
        cm = oracle_mod.unpack_codes(words, bits, D)
        for z in _box_samples(rng, lo, hi, 40):
            w2, m2, a2, _ = oracle_mod.encode_residual_rot(z, ref, bits, group)
            if aok[0]:
                assert a2 == alpha[0]
            c2 = oracle_mod.unpack_codes(w2, bits, D)
            ok = cok.astype(bool)
            assert np.all(c2[ok] == cm[ok])
            assert np.all(m2[mok.astype(bool)] == meta[mok.astype(bool)])


def test_dense_decode_is_attention_over_u_transpose_z(oracle_mod):
    """The rotated-domain decode [RQ App. G.2] equals plain attention over
    X^ = U^T Z^ with the binary16-rounded query, for non-symmetric signed
    permutations (a U / U^T mix-up fails), and reconstruct_dense is U^T Z^."""
    rng = np.random.default_rng(6)
    B, H, T, D = 2, 2, 9, 64
    zk = rng.standard_normal((B, H, T, D))
    zv = rng.standard_normal((B, H, T, D))
    uk = np.stack([_signed_perm(rng, D)[0] for _ in range(H)])
    uv = np.stack([_signed_perm(rng, D)[0] for _ in range(H)])
    q = np.array([oracle_mod.f32_to_bf16_bits(float(v)) for v in rng.standard_normal(B * H * D)],
                 np.uint16).reshape(B, H, D)
    kc = np.array([oracle_mod.f32_to_bf16_bits(float(v)) for v in rng.standard_normal(B * H * D)],
                  np.uint16).reshape(B, H, D)
    vc = kc[:, ::-1].copy()
    seq = [T, 4]
    got = oracle_mod.decode_attention_dense(zk, zv, q, seq, kc, vc, uk, uv)
    ukf = oracle_mod.f16_bits_to_f64(uk)
    uvf = oracle_mod.f16_bits_to_f64(uv)
    khat = np.einsum("hij,bhti->bhtj", ukf, zk)       # U_K^T z per row
    vhat = np.einsum("hij,bhti->bhtj", uvf, zv)
    qf = oracle_mod.bf16_bits_to_f64(q)
    qh = qf.astype(np.float16).astype(np.float64)
    for b in range(B):
        for h in range(H):
            n = seq[b]
            s = np.concatenate([khat[b, h, :n] @ qh[b, h],
                                [qf[b, h] @ oracle_mod.bf16_bits_to_f64(kc[b, h])]]) / np.sqrt(D)
            p = np.exp(s - s.max())
            o = (p[:n] @ vhat[b, h, :n] + p[n] * oracle_mod.bf16_bits_to_f64(vc[b, h])) / p.sum()
            np.testing.assert_allclose(got[b, h], o, rtol=1e-12, atol=1e-12)
    # reconstruct_dense on a lossless-by-construction case: U^T applied per head
    encs = [{"codes": np.zeros((H * T, D // 16), np.uint32),
             "meta": np.tile(np.uint32(0x3C00 << 16), (H * T, D // 32)),
             "alpha": None, "zhat": np.ones((H * T, D), np.float32)}]
    xr = oracle_mod.reconstruct_dense(encs, 0, (2,), (32,), uk, H, T, policy="last")
    ones = np.ones(D)
    for h in range(H):
        np.testing.assert_array_equal(xr[h * T], ukf[h].T @ ones)
