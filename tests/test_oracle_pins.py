"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form, an invariant, a library
routine, brute force on tiny inputs, or a number the ResidualQuant pages print
(tests/golden/pages_storage.txt), chosen so that a dropped term, a wrong sign
or index, or a transposed operand in the oracle fails at least one of them.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                vals[k] = float(v)
    return vals


# ---------------------------------------------------------------- formats --

def _probe_floats(rng, n=4000):
    v = np.concatenate([
        rng.standard_normal(n).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(n) * 1e-5).astype(np.float32),          # fp16 subnormals
        (rng.standard_normal(n) * 1e-8).astype(np.float32),          # flush-to-zero region
        (rng.standard_normal(n) * 3e4).astype(np.float32),           # near fp16 overflow
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 65536.0, 1e30, 6.1e-5, 5.96e-8,
                  2.98e-8, 2.9802322e-08, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11], np.float32),
    ])
    # exact ties of fp16: k + 0.5 ulp patterns
    k = rng.integers(1024, 2048, 200).astype(np.float32)
    ties = ((k + np.float32(0.5)) * np.float32(2.0 ** -10)).astype(np.float32)
    return np.concatenate([v, ties, -ties])


def test_f16_round_trip_matches_numpy(oracle_mod):
    """fp32 -> fp16 (RN-even) and fp16 -> fp32 agree with numpy's IEEE conversions."""
    rng = np.random.default_rng(0)
    v = _probe_floats(rng)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    got = np.array([oracle_mod.f32_to_f16_bits(x) for x in v], np.uint16)
    np.testing.assert_array_equal(got, want)
    allbits = np.arange(0, 1 << 16, 97, dtype=np.uint32).astype(np.uint16)
    ref = allbits.view(np.float16).astype(np.float32)
    mine = np.array([oracle_mod.f16_bits_to_f32(int(b)) for b in allbits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    np.testing.assert_array_equal(mine[~nan], ref[~nan])


def test_bf16_round_trip_matches_torch(oracle_mod):
    rng = np.random.default_rng(1)
    v = _probe_floats(rng)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.f32_to_bf16_bits(x) for x in v], np.uint16)
    np.testing.assert_array_equal(got, want)
    for b in [0x0000, 0x8000, 0x3F80, 0xC2F7, 0x0001, 0x7F7F]:
        assert oracle_mod.bf16_bits_to_f32(b) == float(
            torch.from_numpy(np.array([b], np.uint16).view(np.int16)).view(torch.bfloat16).float()[0])


# --------------------------------------------------------------- rotation --

@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_fwht_equals_scipy_hadamard(oracle_mod, D):
    """H x by the butterfly equals scipy's Sylvester matrix / sqrt(D) times x."""
    rng = np.random.default_rng(D)
    x = rng.standard_normal((5, D)).astype(np.float32)
    H = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    want = x.astype(np.float64) @ H.T
    got = oracle_mod.fwht_f32(x)
    assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want))
    got64 = oracle_mod.fwht_f64(x)
    assert np.max(np.abs(got64 - want)) <= 1e-13 * np.max(np.abs(want))


def test_fwht_sign_pattern_popcount(oracle_mod):
    """Row i of H is (-1)^popcount(i & j) / sqrt(D): transform each basis vector."""
    D = 64
    eye = np.eye(D, dtype=np.float32)
    Ht = oracle_mod.fwht_f32(eye)          # row i = H e_i = column i of H
    i, j = np.meshgrid(np.arange(D), np.arange(D), indexing="ij")
    pc = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    want = np.where(pc % 2 == 0, 1.0, -1.0) / 8.0
    np.testing.assert_array_equal(Ht, want.astype(np.float32))


def test_fwht_involution_exact_d64(oracle_mod):
    """H H^T = I; exact for D=64 on small integers because 1/sqrt(64) = 1/8."""
    rng = np.random.default_rng(2)
    x = rng.integers(-50, 50, (8, 64)).astype(np.float32)
    np.testing.assert_array_equal(oracle_mod.fwht_f32(oracle_mod.fwht_f32(x)), x)
    e0 = np.zeros(64, np.float32)
    e0[0] = 1
    np.testing.assert_array_equal(oracle_mod.fwht_f32(e0), np.full(64, 0.125, np.float32))


def test_row_length_outside_the_buffers_is_refused(oracle_mod):
    """The C row functions hold rows of at most 256 channels: longer or
    non-power-of-two rows raise before any C code runs."""
    for D in (512, 96, 16):
        with pytest.raises(ValueError):
            oracle_mod.quantize(np.zeros(D, np.float32), 2, 16)
        with pytest.raises(ValueError):
            oracle_mod.encode_side(np.zeros((2, 1, D), np.uint16), (2, 4), (16, 16))


def test_rot_scale_is_rounded_inverse_sqrt(oracle_mod):
    for D in (32, 64, 128, 256):
        assert oracle_mod.rot_scale(D) == float(np.float32(1.0 / np.sqrt(np.float64(D))))


def test_rotation_preserves_scores(oracle_mod):
    """q.k = (Hq).(Hk) with quantisation bypassed (orthogonality)."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((16, 128))
    k = rng.standard_normal((16, 128)) * np.exp(0.5 * rng.standard_normal(128))
    s0 = np.sum(q * k, axis=1)
    s1 = np.sum(oracle_mod.fwht_f64(q) * oracle_mod.fwht_f64(k), axis=1)
    assert np.max(np.abs(s1 - s0)) <= 1e-12 * np.max(np.abs(s0))
    s2 = np.sum(oracle_mod.fwht_f32(q).astype(np.float64) * oracle_mod.fwht_f32(k), axis=1)
    assert np.max(np.abs(s2 - s0)) <= 1e-6 * np.sum(np.abs(q) * np.abs(k), axis=1).max()


# ------------------------------------------------------------- dot product --

def test_dot_exact_on_integers(oracle_mod):
    rng = np.random.default_rng(4)
    for D in (32, 64, 128, 256):
        a = rng.integers(-300, 300, D)
        b = rng.integers(-300, 300, D)
        assert oracle_mod.dot_f32(a.astype(np.float32), b.astype(np.float32)) == float(np.dot(a, b))


def test_dot_within_summation_bound(oracle_mod):
    rng = np.random.default_rng(5)
    for D in (64, 128):
        a = rng.standard_normal(D).astype(np.float32)
        b = rng.standard_normal(D).astype(np.float32)
        exact = float(np.dot(a.astype(np.float64), b.astype(np.float64)))
        bound = (D + 8) * 2.0 ** -24 * float(np.sum(np.abs(a.astype(np.float64) * b)))
        assert abs(oracle_mod.dot_f32(a, b) - exact) <= bound
        # swapping the operands cannot change the value
        assert oracle_mod.dot_f32(a, b) == oracle_mod.dot_f32(b, a)


# ------------------------------------------------------------ quantisation --

def test_int2_ramp_uses_all_four_levels(oracle_mod):
    """Affine INT2 has the four levels o, o+s, o+2s, o+3s [RQ §2.1]."""
    o, s = np.float32(-1.25), np.float32(0.5)   # fp16-exact
    z = np.array([o + k * s for k in range(4)] * 8, np.float32)
    words, meta, deq = oracle_mod.quantize(z, 2, 32)
    codes = oracle_mod.unpack_codes(words, 2, 32)
    np.testing.assert_array_equal(codes, np.tile(np.arange(4), 8))
    sc, zz = oracle_mod.meta_scale_zero(meta)
    assert sc[0] == s and zz[0] == o
    np.testing.assert_array_equal(deq, z)


def test_packing_bit_positions():
    """Storage order (hand-computed words): 2-bit channel i -> word i/16, bits
    2*(i%16); 4-bit channel 16u+v -> word 2u+((v>>1)&1), nibble 2*(v>>2)+(v&1)."""
    import oracle
    o = np.float32(0.0)
    # INT4, 32 channels with codes 0..15 then 15..0, scale 1, offset 0:
    # word 0 holds channels 0,1,4,5,8,9,12,13 in nibbles 0..7, word 1 the rest.
    z = np.array(list(range(16)) + list(range(15, -1, -1)), np.float32)
    words, _, _ = oracle.quantize(z, 4, 32)
    assert [hex(w) for w in words] == ["0xdc985410", "0xfeba7632", "0x2367abef", "0x14589cd"]
    # INT2, 16 channels: codes 3,0,1,2,... -> ((3)|(0<<2)|(1<<4)|(2<<6)) per byte = 0x93
    z2 = np.array([3, 0, 1, 2] * 4 + [0, 0, 0, 3] * 4, np.float32) + o
    w2, _, _ = oracle.quantize(z2, 2, 32)
    assert [hex(w) for w in w2] == ["0x93939393", "0xc0c0c0c0"]


def _tie_distance(u):
    return np.abs(np.abs(u - np.floor(u)) - 0.5)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 32), (2, 16), (2, 64), (4, 64)])
def test_codes_are_nearest_level_brute_force(oracle_mod, bits, group):
    """Brute force over every level: the code is the nearest level (clamped),
    except where the scaled value sits within 1e-4 of a half-way tie."""
    rng = np.random.default_rng(bits * 100 + group)
    qmax = (1 << bits) - 1
    checked = 0
    for trial in range(40):
        z = (rng.standard_normal(128) * rng.uniform(0.01, 5)).astype(np.float32)
        words, meta, deq = oracle_mod.quantize(z, bits, group)
        codes = oracle_mod.unpack_codes(words, bits, 128).astype(np.int64)
        sc, zz = oracle_mod.meta_scale_zero(meta)
        for gi in range(128 // group):
            sl = slice(gi * group, (gi + 1) * group)
            zg = z[sl].astype(np.float64)
            s, o = float(sc[gi]), float(zz[gi])
            # metadata: fp16 of (max-min)/qmax and of min
            assert sc[gi] == np.float16(np.float32(np.float32(zg.max() - zg.min()) / qmax))
            assert zz[gi] == np.float16(np.float32(zg.min()))
            levels = o + s * np.arange(qmax + 1)
            best = np.argmin(np.abs(zg[:, None] - levels[None, :]), axis=1)
            u = (zg - o) / s
            ok = _tie_distance(np.clip(u, 0, qmax)) > 1e-4
            np.testing.assert_array_equal(codes[sl][ok], best[ok])
            checked += ok.sum()
            # the group's extremes land on the end codes
            assert codes[sl][np.argmin(zg)] == 0 and codes[sl][np.argmax(zg)] == qmax
            # every dequantised value is a level, within fp32 rounding of fma
            np.testing.assert_allclose(deq[sl], levels[codes[sl]], rtol=0, atol=2e-7 * (abs(o) + s * qmax))
            assert np.all(np.abs(zg - levels[codes[sl]]) <= 0.5 * s * (1 + 1e-3) + 1e-3 * s)
    assert checked > 1000


def test_constant_group_codes_zero(oracle_mod):
    z = np.full(64, 0.8125, np.float32)
    words, meta, deq = oracle_mod.quantize(z, 2, 32)
    assert np.all(words == 0)
    sc, zz = oracle_mod.meta_scale_zero(meta)
    assert np.all(sc == 0) and np.all(zz == np.float32(0.8125))
    np.testing.assert_array_equal(deq, z)


# ---------------------------------------------------------- LS coefficient --

def _anchor_row(oracle_mod, seed, D=128):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(D).astype(np.float32)
    _, _, A = oracle_mod.quantize(z, 4, 32)
    return A


@pytest.mark.parametrize("c", [1.0, 0.5, 2.0, -0.25, 4.0])
def test_scaled_reference_gives_alpha_c_and_zero_residual(oracle_mod, c):
    """X_r = c R^ gives alpha = c and a zero residual [RQ §3.2, App. G.1]."""
    A = _anchor_row(oracle_mod, 7)
    z = (np.float32(c) * A).astype(np.float32)
    words, meta, ab, zhat = oracle_mod.encode_residual_rot(z, A, 2, 32)
    assert oracle_mod.bf16_bits_to_f32(ab) == c
    assert np.all(words == 0)
    sc, zz = oracle_mod.meta_scale_zero(meta)
    assert np.all(sc == 0) and np.all(zz == 0)
    np.testing.assert_array_equal(zhat, z)


def test_alpha_is_bf16_of_least_squares(oracle_mod):
    """alpha~ is the bf16 rounding of argmin_a ||z - a ref||^2 (within one bf16 step)."""
    rng = np.random.default_rng(8)
    for seed in range(30):
        A = _anchor_row(oracle_mod, 100 + seed)
        c = rng.uniform(0.7, 1.3)
        z = (c * A + 0.3 * rng.standard_normal(128)).astype(np.float32)
        _, _, ab, _ = oracle_mod.encode_residual_rot(z, A, 2, 32)
        a64 = np.dot(z.astype(np.float64), A) / np.dot(A.astype(np.float64), A)
        got = oracle_mod.bf16_bits_to_f32(ab)
        assert abs(got - a64) <= 2.0 ** -8 * abs(a64)


def test_zero_anchor_gives_alpha_zero(oracle_mod):
    rng = np.random.default_rng(9)
    z = rng.standard_normal(128).astype(np.float32)
    ref = np.zeros(128, np.float32)
    words, meta, ab, zhat = oracle_mod.encode_residual_rot(z, ref, 2, 32)
    assert ab == 0
    w2, m2, d2 = oracle_mod.quantize(z, 2, 32)
    np.testing.assert_array_equal(words, w2)
    np.testing.assert_array_equal(meta, m2)
    np.testing.assert_array_equal(zhat, d2)


def test_residual_beats_direct_quantisation(oracle_mod):
    """The point of the method: on correlated loops, anchor + LS residual at INT2
    reconstructs better than direct INT2 of the same loop [RQ §3.1, §3.2]."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=64)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_K, l, [0], [0, 1], 0, 64)).reshape(-1, 128)
                  for l in range(4)])
    encs = oracle_mod.encode_side(x, w.bits, w.group)
    xs = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for r in range(3):
        rec = oracle_mod.reconstruct(encs, r, w.bits, w.group)
        direct = oracle_mod.encode_side(x[r:r + 1], (2,), (32,))
        rec_d = oracle_mod.reconstruct(direct, 0, (2,), (32,))
        err_res = np.sum((rec - xs[r]) ** 2)
        err_dir = np.sum((rec_d - xs[r]) ** 2)
        assert err_res < 0.5 * err_dir


def test_chained_equals_shared_next_to_anchor(oracle_mod):
    """Loop L-2 references the anchor under both policies: identical encodings;
    the chain differs further away [RQ §5.2, App. D]."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["huginn_deep"].replace(batch=1, heads=1, tokens=16)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_V, l, [0], [0], 0, 16)).reshape(-1, 128)
                  for l in range(w.loops)])
    es = oracle_mod.encode_side(x, w.bits, w.group, "last")
    ec = oracle_mod.encode_side(x, w.bits, w.group, "next")
    r = w.loops - 2
    for k in ("codes", "meta", "alpha"):
        np.testing.assert_array_equal(es[r][k], ec[r][k])
    assert not np.array_equal(es[0]["codes"], ec[0]["codes"])
    # the chained reconstruction of loop r equals alpha_r * (reconstruction of r+1) + D(c_r)
    z1 = oracle_mod.reconstruct_rotated(ec, 1, w.bits, w.group, "next")
    z0 = oracle_mod.reconstruct_rotated(ec, 0, w.bits, w.group, "next")
    lv = oracle_mod._levels_f64(ec[0], w.bits[0], w.group[0], 128)
    a0 = oracle_mod.bf16_bits_to_f64(ec[0]["alpha"])[:, None]
    np.testing.assert_allclose(z0, a0 * z1 + lv, rtol=0, atol=1e-12)


def _exact_multiple_chain(mults):
    """Three loops on an exact grid at D = 64 (fp32(1/sqrt(64)) = 1/8 exactly):
    x = a (e_0 + e_1) rotates to Z = a/8 on even channels and 0 on odd ones,
    so an INT4 anchor with a = 60 spans the levels 0 .. 15 with scale 1 and
    offset 0 and is stored exactly.  Loop l is x scaled by mults[l]; every
    product stays bf16-exact."""
    D = 64
    x = np.zeros((3, 1, D), np.float32)
    for l, m in enumerate(mults):
        x[l, 0, 0] = x[l, 0, 1] = 60.0 * m
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), x)
    return bits


@pytest.mark.parametrize("policy,mults,alphas", [
    # Next-loop: anchor = loop 2; loop 1 = 3 x loop 2, loop 0 = 2 x loop 1
    ("next", (6.0, 3.0, 1.0), {1: 3.0, 0: 2.0}),
    # Previous-loop (the mirror): anchor = loop 0; loop 1 = 3 x loop 0, loop 2 = 2 x loop 1
    ("previous", (1.0, 3.0, 6.0), {1: 3.0, 2: 2.0}),
])
def test_chain_references_on_an_exact_grid(oracle_mod, policy, mults, alphas):
    """Closed form of the reference chain [RQ §3.2, App. D]: with every loop an
    exact multiple of its neighbour toward the anchor, each stored LS
    coefficient is the ratio to that neighbour (3, then 2), every residual is
    exactly zero and the reconstruction reproduces each loop exactly.  A chain
    that referenced the anchor, or the loop two steps away, would store 6 for
    the far loop instead of 2."""
    bits, group = (4, 2, 4), (32, 32, 32)
    if policy == "previous":
        bits = (4, 2, 2)
    encs = oracle_mod.encode_side(_exact_multiple_chain(mults), bits, group, policy)
    anchor = oracle_mod.anchor_loop(3, policy)
    z_anchor = np.zeros(64)
    z_anchor[0::2] = 15.0
    for r, a in alphas.items():
        assert oracle_mod.bf16_bits_to_f32(int(encs[r]["alpha"][0])) == a
        assert not encs[r]["codes"].any() and not encs[r]["meta"].any()
    for r in range(3):
        z = oracle_mod.reconstruct_rotated(encs, r, bits, group, policy)
        np.testing.assert_array_equal(z[0], mults[r] / mults[anchor] * z_anchor)


def test_encoder_reference_row_matches_reconstruction(oracle_mod):
    """The fp32 reconstructed row the encoder keeps (zhat) equals the fp64
    reconstruction from the stored codes, alpha and metadata to fp32 rounding."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=1, tokens=32)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_K, l, [0], [0], 0, 32)).reshape(-1, 128)
                  for l in range(4)])
    encs = oracle_mod.encode_side(x, w.bits, w.group)
    for r in range(4):
        z = oracle_mod.reconstruct_rotated(encs, r, w.bits, w.group)
        np.testing.assert_allclose(encs[r]["zhat"], z, rtol=2e-6, atol=2e-6)


# --------------------------------------------------------------- attention --

def _softmax_attention_numpy(q, K, V, kc, vc, scale):
    s = np.concatenate([K @ q, [kc @ q]]) * scale
    p = np.exp(s - s.max())
    p /= p.sum()
    return p[:-1] @ V + p[-1] * vc


def test_attention_matches_brute_force(oracle_mod):
    rng = np.random.default_rng(10)
    for T in (0, 1, 5, 37):
        q, kc, vc = (rng.standard_normal(64) for _ in range(3))
        K = rng.standard_normal((T, 64)) * 2
        V = rng.standard_normal((T, 64))
        got = oracle_mod.attention(q, K, V, kc, vc, 0.125)
        want = _softmax_attention_numpy(q, K, V, kc, vc, 0.125)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_special_cases(oracle_mod):
    rng = np.random.default_rng(11)
    kc, vc = rng.standard_normal(128), rng.standard_normal(128)
    # no past tokens: the current value alone
    np.testing.assert_allclose(oracle_mod.attention(rng.standard_normal(128), np.zeros((0, 128)),
                                                    np.zeros((0, 128)), kc, vc, 0.1), vc, rtol=1e-15)
    # a zero query gives equal scores: the mean of all values
    V = rng.standard_normal((9, 128))
    got = oracle_mod.attention(np.zeros(128), rng.standard_normal((9, 128)), V, kc, vc, 0.1)
    np.testing.assert_allclose(got, (V.sum(0) + vc) / 10, rtol=1e-12, atol=1e-14)


def test_decode_units_are_independent(oracle_mod):
    """Batch/head units do not interact: permuting heads permutes outputs."""
    rng = np.random.default_rng(12)
    B, H, T, D = 2, 3, 11, 64
    kh, vh = rng.standard_normal((B, H, T, D)), rng.standard_normal((B, H, T, D))
    bf = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, kc, vc = (bf(rng.standard_normal((B, H, D))) for _ in range(3))
    out = oracle_mod.decode_attention(kh, vh, q, [T, 7], kc, vc)
    perm = [2, 0, 1]
    out2 = oracle_mod.decode_attention(kh[:, perm], vh[:, perm], q[:, perm], [T, 7], kc[:, perm],
                                       vc[:, perm])
    np.testing.assert_array_equal(out2, out[:, perm])


# ---------------------------------------------------- storage and accesses --

def test_effective_bits_match_pages():
    """With the pages' 16-bit metadata per group, the accounting reproduces
    every printed b_eff, the alpha overhead and the storage fractions."""
    import oracle
    g = _golden("pages_storage.txt")
    D = 128
    cfgs = {
        "int2_g32": ((2, 2, 2, 2), (32, 32, 32, 32)),
        "int2_g16": ((2, 2, 2, 2), (16, 16, 16, 16)),
        "int24_g32": ((2, 2, 2, 4), (32, 32, 32, 32)),
        "int24_g16": ((2, 2, 2, 4), (16, 16, 16, 32)),   # INT4 keeps g=32 [RQ §5.2]
    }
    for name, (bits, grp) in cfgs.items():
        direct = oracle.effective_bits(bits, grp, D, 16, False)
        resid = oracle.effective_bits(bits, grp, D, 16, True)
        assert round(direct, 1) == g[f"beff_direct_{name}"], name
        assert round(resid, 1) == g[f"beff_residual_{name}"], name
    over = oracle.effective_bits((2,) * 4, (32,) * 4, D, 16, True) - oracle.effective_bits(
        (2,) * 4, (32,) * 4, D, 16, False)
    assert round(over, 3) == g["alpha_overhead_bits"]
    b_rq = oracle.effective_bits((2, 2, 2, 4), (32,) * 4, D, 16, True)
    assert round(b_rq / 16, 3) == g["storage_frac_int24_residual_g32"]
    assert round(oracle.effective_bits((2,) * 4, (32,) * 4, D, 16, False) / 16, 3) == g[
        "storage_frac_int2_direct_g32"]
    assert round(1 - b_rq / 16, 3) == g["storage_reduction_int24"]
    assert round(16 / b_rq, 1) == g["storage_ratio_int24"]


def test_component_reads_match_pages():
    import oracle
    g = _golden("pages_storage.txt")
    assert oracle.component_reads(4, True) == g["reads_chained_L4"]
    assert oracle.component_reads(4, False) == g["reads_shared_L4"]
    assert oracle.component_reads(32, True) == g["reads_chained_L32"]
    assert oracle.component_reads(32, False) == g["reads_shared_L32"]
    assert round(oracle.component_reads(4, True) / oracle.component_reads(4, False), 2) == g[
        "reads_ratio_L4"]
    assert round(oracle.component_reads(32, True) / oracle.component_reads(32, False), 2) == g[
        "reads_ratio_L32"]
    assert 8 * oracle.component_reads(4, True) == g["reads_chained_huginn_8x4"]
    assert 8 * oracle.component_reads(4, False) == g["reads_shared_huginn_8x4"]
    # closed forms L(L+1)/2 and 2L-1 for every L
    for L in range(1, 40):
        assert oracle.component_reads(L, True) == L * (L + 1) // 2
        assert oracle.component_reads(L, False) == 2 * L - 1


# ------------------------------------------- First-loop / Previous-loop [RQ §3.2]

def _synthetic_loops(w, side, T=24):
    import residual_bit_kv_b200.synth as synth
    return np.stack([synth.bits_of(synth.kv(w, 0, side, l, [0], [0], 0, T)).reshape(-1, w.head_dim)
                     for l in range(w.loops)])


@pytest.mark.parametrize("pol,mirror", [("first", "last"), ("previous", "next")])
def test_first_and_previous_mirror_last_and_next(oracle_mod, pol, mirror):
    """First-loop (Previous-loop) is Last-loop (Next-loop) with the loop order
    reversed: the anchor moves to loop 0 and the references point down the
    loop index instead of up [RQ §3.2, App. D].  Encoding the reversed loops
    under the mirrored policy stores identical bits, and reconstructs
    identically."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["huginn_deep"].replace(loops=5, bits=(4, 2, 2, 4, 2),
                                               group=(32, 64, 16, 32, 64),
                                               sigma=(0.4, 0.3, 0.2, 0.1))
    x = _synthetic_loops(w, synth.SIDE_K)
    L = w.loops
    e = oracle_mod.encode_side(x, w.bits, w.group, pol)
    m = oracle_mod.encode_side(x[::-1], w.bits[::-1], w.group[::-1], mirror)
    assert oracle_mod.anchor_loop(L, pol) == 0 and e[0]["alpha"] is None
    for r in range(L):
        for k in ("codes", "meta", "alpha"):
            if e[r][k] is None:
                assert m[L - 1 - r][k] is None
            else:
                np.testing.assert_array_equal(e[r][k], m[L - 1 - r][k])
        np.testing.assert_array_equal(
            oracle_mod.reconstruct_rotated(e, r, w.bits, w.group, pol),
            oracle_mod.reconstruct_rotated(m, L - 1 - r, w.bits[::-1], w.group[::-1], mirror))


def test_previous_loop_chain_is_the_recursion(oracle_mod):
    """Previous-loop: loop r is rebuilt from loop r-1's reconstruction,
    Z^_r = alpha~_r Z^_{r-1} + D(c_r), down to the first-loop anchor."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"]
    x = _synthetic_loops(w, synth.SIDE_V)
    e = oracle_mod.encode_side(x, w.bits[::-1], w.group[::-1], "previous")
    bits, group = w.bits[::-1], w.group[::-1]
    for r in range(1, w.loops):
        zr = oracle_mod.reconstruct_rotated(e, r, bits, group, "previous")
        zp = oracle_mod.reconstruct_rotated(e, r - 1, bits, group, "previous")
        lv = oracle_mod._levels_f64(e[r], bits[r], group[r], w.head_dim)
        a = oracle_mod.bf16_bits_to_f64(e[r]["alpha"])[:, None]
        np.testing.assert_allclose(zr, a * zp + lv, rtol=0, atol=1e-12)


def test_unit_alpha_residual_closed_form(oracle_mod):
    """Without LS scaling alpha = 1 [RQ §3.1-§3.2]: a loop equal to twice the
    anchor, whose rotation hits the INT4 levels exactly (integers 0..15 with
    s~ = 1, z~ = 0), leaves the residual E = 2Z - Z = Z; INT2 then takes
    s~ = 15/3 = 5, z~ = 0 and codes rint(Z/5), and the loop is rebuilt as
    Z + 5 rint(Z/5).  LS scaling instead finds alpha = 2 and a zero residual."""
    D = 64
    rng = np.random.default_rng(7)
    Z = rng.integers(0, 16, size=D).astype(np.float64)
    Z[0], Z[1], Z[32], Z[33] = 0, 15, 0, 15            # every group spans [0, 15]
    H = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    xa = H @ Z                                          # exact multiples of 1/8
    assert np.all(xa * 8 == np.round(xa * 8)) and np.max(np.abs(xa)) < 64
    xa_b = torch.tensor(xa, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(xa_b.float().numpy().astype(np.float64), xa)
    xb = synth_bits(xa_b)
    x = np.stack([synth_bits(xa_b * 2), xb])[:, None, :]   # loop 0 = 2 x anchor, loop 1 = anchor
    bits, group = (2, 4), (32, 32)
    unit = oracle_mod.encode_side(x, bits, group, "last", unit_alpha=True)
    ls = oracle_mod.encode_side(x, bits, group, "last")
    assert np.all(unit[0]["alpha"] == 0x3F80)           # bf16(1.0)
    assert np.all(ls[0]["alpha"] == 0x4000)             # bf16(2.0)
    assert np.all(ls[0]["codes"] == 0) and np.all(ls[0]["meta"] == 0)
    codes = oracle_mod.unpack_codes(unit[0]["codes"], 2, D).reshape(D)
    np.testing.assert_array_equal(codes, np.round(Z / 5))
    s, z = oracle_mod.meta_scale_zero(unit[0]["meta"])
    np.testing.assert_array_equal(s.reshape(-1), [5.0, 5.0])
    np.testing.assert_array_equal(z.reshape(-1), [0.0, 0.0])
    rec = oracle_mod.reconstruct_rotated(unit, 0, bits, group, "last").reshape(D)
    np.testing.assert_array_equal(rec, Z + 5 * np.round(Z / 5))


def synth_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------- 16-bit metadata per group --
# The pages count 16 bits of scale and offset per group [RQ §5.1, App. A.3]
# without fixing a format; the variant here is a scale byte (unsigned e5m3)
# and an offset byte (a multiple of scale/8).

def _m8_value(b):
    """The scale byte's value from its definition, in exact fp64."""
    E, m = b >> 3, b & 7
    return 0.0 if E == 0 else (1 + m / 8) * 2.0 ** (E - 18)


def test_m8_scale_byte_table_and_round_trip(oracle_mod):
    assert oracle_mod.M8_BIAS == 18
    for b in range(256):
        v = oracle_mod.m8_scale_decode(b)
        assert v == _m8_value(b), b
        if b >> 3:
            assert oracle_mod.m8_scale_encode(v) == b, b
    assert oracle_mod.m8_scale_encode(0.0) == 0 and oracle_mod.m8_scale_encode(-1.0) == 0
    assert oracle_mod.m8_scale_encode(float("nan")) == 0


def test_m8_scale_is_nearest_brute_force(oracle_mod):
    """Every positive input goes to the nearest representable value (ties to
    the even m), below the range to the smallest, above it to the largest."""
    vals = np.array([_m8_value(b) for b in range(8, 256)])
    rng = np.random.default_rng(11)
    s = np.float32(2.0) ** rng.uniform(-20, 15, 3000).astype(np.float32)
    # exact midpoints between neighbours (ties)
    mids = ((vals[:-1] + vals[1:]) / 2)
    mids = mids[np.float32(mids) == mids].astype(np.float32)
    for x in np.concatenate([s, mids]):
        x = float(x)
        b = oracle_mod.m8_scale_encode(x)
        got = _m8_value(b)
        if x < vals[0]:
            assert b == 0x08
            continue
        if x > vals[-1]:
            assert b == 0xFF
            continue
        d = np.abs(vals - x)
        best = d.min()
        assert abs(got - x) == best, (x, got)
        if (d == best).sum() == 2:      # a tie: the even mantissa wins
            assert (b & 7) % 2 == 0, (x, b)


def test_m8_ramp_uses_all_four_levels(oracle_mod):
    """Scale 1 and offset -1.5 are exact in the bytes: the INT2 ramp
    -1.5, -0.5, 0.5, 1.5 gets codes 0..3 and dequantises exactly."""
    z = np.array([-1.5, -0.5, 0.5, 1.5] * 8, np.float32)
    words, meta, deq = oracle_mod.quantize_m8(z, 2, 32)
    np.testing.assert_array_equal(oracle_mod.unpack_codes(words, 2, 32), np.tile(np.arange(4), 8))
    assert meta[0] & 0xFF == oracle_mod.m8_scale_encode(1.0)
    assert np.int8(np.uint8(meta[0] >> 8)) == -12
    np.testing.assert_array_equal(deq, z)


@pytest.mark.parametrize("bits,group", [(2, 16), (2, 32), (2, 64), (4, 32), (4, 128)])
def test_m8_codes_are_nearest_level_brute_force(oracle_mod, bits, group):
    """Metadata from its definition; every code the nearest level of the
    grid z~ + k s~ (clamped), away from half-way ties; z~ <= mn < z~ + s~/8
    while the offset byte is not saturated."""
    rng = np.random.default_rng(bits * 1000 + group)
    qmax = (1 << bits) - 1
    checked = 0
    for trial in range(40):
        z = (rng.standard_normal(128) * rng.uniform(0.01, 5) +
             rng.uniform(-1, 1) * (trial % 3)).astype(np.float32)
        words, meta, deq = oracle_mod.quantize_m8(z, bits, group)
        codes = oracle_mod.unpack_codes(words, bits, 128).astype(np.int64)
        for gi in range(128 // group):
            sl = slice(gi * group, (gi + 1) * group)
            zg = z[sl]
            mn, mx = np.float32(zg.min()), np.float32(zg.max())
            s0 = np.float32(np.float32(mx - mn) / np.float32(qmax))
            s1 = np.float32(np.float32(abs(mn)) / np.float32(15.875))
            sb = int(meta[gi]) & 0xFF
            zq = int(np.int8(np.uint8(int(meta[gi]) >> 8)))
            assert sb == oracle_mod.m8_scale_encode(float(max(s0, s1)))
            s = _m8_value(sb)
            o = zq * s / 8
            t = np.floor(np.float32(np.float32(8) * mn) / np.float32(s))
            if -128 <= t <= 127:
                assert zq == t and o <= mn < o + s / 8
            levels = o + s * np.arange(qmax + 1)
            best = np.argmin(np.abs(zg[:, None].astype(np.float64) - levels[None, :]), axis=1)
            u = (zg.astype(np.float64) - o) / s
            ok = _tie_distance(np.clip(u, 0, qmax)) > 1e-4
            np.testing.assert_array_equal(codes[sl][ok], best[ok])
            checked += ok.sum()
            np.testing.assert_array_equal(deq[sl], np.float32(levels[codes[sl]]))
    assert checked > 1000


def test_m8_constant_group_keeps_its_value(oracle_mod):
    """A constant nonzero group (zero range) is still reproduced: the scale
    becomes |c| / 15.875 (rounded to nearest, or one step up where the
    offset byte would otherwise saturate) and the level nearest to c is
    within half a step; a zero group stays exactly zero."""
    for c in (3.0, -0.7, 1e-3, -250.0):
        z = np.full(32, c, np.float32)
        words, meta, deq = oracle_mod.quantize_m8(z, 2, 32)
        s = _m8_value(int(meta[0]) & 0xFF)
        assert abs(c) / 15.875 * (1 - 1 / 17) <= s <= abs(c) / 15.875 * (1 + 1 / 16) * (1 + 1 / 8)
        assert np.all(np.abs(deq - c) <= s / 2 + 1e-6 * abs(c))
    words, meta, deq = oracle_mod.quantize_m8(np.zeros(32, np.float32), 2, 32)
    assert meta[0] == 0 and not deq.any() and not words.any()


def test_m8_error_close_to_fp16_metadata(oracle_mod):
    """Design check on rotated synthetic rows: halving the metadata costs at
    most 10% (INT2) / 15% (INT4) more squared error than fp16 scale + fp16
    offset, and the offset byte never saturates on this data."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"]
    x = synth.kv_full(w, 0, 0, 1, 0, 32, device="cpu").float().numpy().reshape(-1, 128)[:512]
    Z = oracle_mod.fwht_f32(x.astype(np.float32))
    for bits, lim in ((2, 1.10), (4, 1.15)):
        e16 = e8 = 0.0
        for row in Z:
            e16 += float(((oracle_mod.quantize(row, bits, 32)[2] - row) ** 2).sum())
            words, meta, deq = oracle_mod.quantize_m8(row, bits, 32)
            e8 += float(((deq - row) ** 2).sum())
            zq = (meta >> 8).astype(np.uint8).view(np.int8)
            assert np.all((zq > -128) & (zq < 127))
        assert e8 <= lim * e16, (bits, e8 / e16)


@pytest.mark.parametrize("bits", [2, 4])
def test_m8_error_bound_and_offset_range(oracle_mod, bits):
    """Worst case of the 16-bit-metadata quantiser: every value lies within
    max(1/2, (2^b - 1)/16 + 1/8) steps s~ of its level (s~ at most 1/17
    below the range scale, z~ at most s~/8 below the minimum), and the
    offset byte never saturates while the scale is inside the byte's range.
    Rows: normal, shifted, one-sided narrow groups (offset far from zero)
    and rows whose range scale sits just below a rounding midpoint."""
    qmax = (1 << bits) - 1
    bound = max(0.5, qmax / 16 + 1 / 8)
    rng = np.random.default_rng(40 + bits)
    rows = [rng.standard_normal(128) * 2.0,
            rng.standard_normal(128) * 0.3 + 5.0,
            rng.uniform(20.0, 20.5, 128),
            -rng.uniform(7.0, 7.2, 128)]
    for k in range(40):
        # range scale (1 + 1/16)(1 - eps) 2^e rounds down to 2^e; minimum just
        # below a multiple of s~/8 above zero
        e = int(rng.integers(-6, 4))
        s0 = (1 + 1 / 16) * (1 - 2.0 ** -20) * 2.0 ** e
        mn = (int(rng.integers(0, 40)) + 0.999) * 2.0 ** e / 8
        g = np.full(32, mn)
        g[1] = mn + qmax * s0
        g[2:] = mn + rng.uniform(0, qmax * s0, 30)
        rows.append(np.tile(g, 4))
    worst = 0.0
    for z in rows:
        z = z.astype(np.float32)
        for group in (16, 32, 64, 128):
            words, meta, deq = oracle_mod.quantize_m8(z, bits, group)
            for j in range(128 // group):
                s = _m8_value(int(meta[j]) & 0xFF)
                zq = int(np.int8(np.uint8(int(meta[j]) >> 8)))
                assert -128 < zq < 127 or (int(meta[j]) & 0xFF) == 0xFF
                err = np.max(np.abs(deq[j * group:(j + 1) * group].astype(np.float64) -
                                    z[j * group:(j + 1) * group]))
                assert err <= bound * s * (1 + 2 ** -20) + 1e-6 * np.max(np.abs(z)), (group, err / s)
                worst = max(worst, err / s)
    if bits == 4:
        assert worst > 1.0   # the INT4 bound is reached: more than one step at a group's top
    else:
        assert worst <= 0.5 + 1e-6


def test_m8_levels_follow_the_byte_definitions(oracle_mod):
    """The fp64 levels of 16-bit-metadata rows are s~ c + zq s~ / 8 with s~
    read off the scale byte's definition, and match the quantiser's fp32
    levels to one fp32 rounding."""
    rng = np.random.default_rng(21)
    for bits, group in ((2, 32), (4, 32), (2, 16), (4, 64)):
        z = (rng.standard_normal((6, 128)) * 2).astype(np.float32)
        rows = [oracle_mod.quantize_m8(r, bits, group) for r in z]
        enc = {"codes": np.stack([r[0] for r in rows]), "meta": np.stack([r[1] for r in rows])}
        lv = oracle_mod._levels_f64(enc, bits, group, 128)
        codes = oracle_mod.unpack_codes(enc["codes"], bits, 128).astype(np.float64)
        for n in range(6):
            for i in range(128):
                m = int(enc["meta"][n, i // group])
                s = _m8_value(m & 0xFF)
                zq = int(np.int8(np.uint8(m >> 8)))
                assert lv[n, i] == s * codes[n, i] + zq * s / 8
            np.testing.assert_allclose(rows[n][2], lv[n], rtol=2 ** -24, atol=0)


@pytest.mark.parametrize("c", [1.0, 0.5, -0.25, 4.0])
def test_m8_scaled_reference_gives_alpha_c_and_zero_residual(oracle_mod, c):
    """With 16-bit metadata too, X_r = c R^ gives alpha = c, a zero residual
    (all-zero codes and metadata) and Z^_r = X_r [RQ §3.2, App. G.1]."""
    rng = np.random.default_rng(7)
    _, _, A = oracle_mod.quantize_m8(rng.standard_normal(128).astype(np.float32), 4, 32)
    z = (np.float32(c) * A).astype(np.float32)
    words, meta, ab, zhat = oracle_mod.encode_residual_rot_m8(z, A, 2, 32)
    assert oracle_mod.bf16_bits_to_f32(ab) == c
    assert not words.any() and not meta.any()
    np.testing.assert_array_equal(zhat, z)


def test_m8_side_encoding_invariants(oracle_mod):
    """encode_side with 16-bit metadata: Last-loop and Next-loop agree next to
    the anchor; every kept reference row equals the fp64 reconstruction from
    the stored data to fp32 rounding; the reconstruction error stays within
    10% of the fp16-metadata encoding's."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=64)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_K, l, [0], [0, 1], 0, 64)).reshape(-1, 128)
                  for l in range(w.loops)])
    es = oracle_mod.encode_side(x, w.bits, w.group, "last", meta16=True)
    ec = oracle_mod.encode_side(x, w.bits, w.group, "next", meta16=True)
    r = w.loops - 2
    for k in ("codes", "meta", "alpha"):
        np.testing.assert_array_equal(es[r][k], ec[r][k])
    assert es[0]["meta"].dtype == np.uint16
    e16 = oracle_mod.encode_side(x, w.bits, w.group, "last")
    xr = oracle_mod.fwht_f64(oracle_mod.bf16_bits_to_f64(x))
    for loop in range(w.loops):
        z = oracle_mod.reconstruct_rotated(es, loop, w.bits, w.group)
        np.testing.assert_allclose(es[loop]["zhat"], z, rtol=2e-6, atol=2e-6)
        err8 = float(((z - xr[loop]) ** 2).sum())
        err16 = float(((oracle_mod.reconstruct_rotated(e16, loop, w.bits, w.group) - xr[loop]) ** 2).sum())
        assert err8 <= 1.10 * err16, (loop, err8 / err16)


# ------------------------------------------------------ fixed mean mu_r --
# Z^_r = alpha_r A + D(c_r) + mu_r [RQ App. G.2]; the mean is a fixed
# per-loop vector in the rotated domain (not stored per token).

@pytest.mark.parametrize("meta16", [False, True])
@pytest.mark.parametrize("policy", ["last", "next", "first", "previous"])
def test_zero_mean_is_the_plain_encoder(oracle_mod, policy, meta16):
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=2, tokens=32)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_V, l, [0], [0, 1], 0, 32)).reshape(-1, 128)
                  for l in range(w.loops)])
    e0 = oracle_mod.encode_side(x, w.bits, w.group, policy, meta16=meta16)
    em = oracle_mod.encode_side(x, w.bits, w.group, policy, meta16=meta16,
                                mu=np.zeros((w.loops,) + x.shape[1:], np.float32))
    for a, b in zip(e0, em):
        for k in ("codes", "meta", "alpha"):
            if a[k] is None:
                assert b[k] is None
            else:
                np.testing.assert_array_equal(a[k], b[k])
        np.testing.assert_array_equal(a["zhat"], b["zhat"])


@pytest.mark.parametrize("meta16", [False, True])
def test_mean_shift_invariance_on_an_exact_grid(oracle_mod, meta16):
    """With every sum exact (values on a 2^-10 grid), encoding z + mu with
    mean mu stores exactly what encoding z without a mean stores, and its
    reconstruction is the mean-free one plus mu."""
    rng = np.random.default_rng(31)
    A = _anchor_row(oracle_mod, 5)
    for trial in range(20):
        z = (np.round(rng.standard_normal(128) * 512) / 1024).astype(np.float32)
        mu = (np.round(rng.uniform(-1, 1, 128) * 1024) / 1024).astype(np.float32)
        w0, m0, a0, zh0 = oracle_mod.encode_residual_rot_ex(z, A, None, 2, 32, meta16=meta16)
        w1, m1, a1, zh1 = oracle_mod.encode_residual_rot_ex(z + mu, A, mu, 2, 32, meta16=meta16)
        assert a0 == a1
        np.testing.assert_array_equal(w0, w1)
        np.testing.assert_array_equal(m0, m1)
        np.testing.assert_array_equal(zh1, (zh0 + mu).astype(np.float32))


@pytest.mark.parametrize("policy", ["last", "next", "previous"])
def test_mean_reconstruction_matches_the_kept_rows(oracle_mod, policy):
    """The fp32 rows the encoder keeps equal the fp64 reconstruction
    alpha~ Z^_ref + D(c) + mu from the stored data (fp32 rounding)."""
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["ouro_layer"].replace(batch=1, heads=1, tokens=64)
    x = np.stack([synth.bits_of(synth.kv(w, 0, synth.SIDE_K, l, [0], [0], 0, 64)).reshape(-1, 128)
                  for l in range(w.loops)])
    rng = np.random.default_rng(32)
    mu = np.broadcast_to(rng.standard_normal((w.loops, 1, 128)).astype(np.float32),
                         (w.loops,) + x.shape[1:]).copy()
    encs = oracle_mod.encode_side(x, w.bits, w.group, policy, mu=mu)
    for r in range(w.loops):
        z = oracle_mod.reconstruct_rotated(encs, r, w.bits, w.group, policy, mu=mu)
        np.testing.assert_allclose(encs[r]["zhat"], z, rtol=2e-6, atol=2e-6)
