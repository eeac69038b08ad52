"""A decode input whose value weights leave the fast decode kernel's
accumulator range in one (batch, head) unit and not in the other.

Head dim 64 (fp32(1/sqrt(64)) = 1/8 exactly), two loops (residual INT2, anchor
INT4, g 32, Last-loop).  Batch row 0, V side: the anchor row of token t is
x = 60 m_t (e_0 + e_1) with m_t = 1024 * 2^(t % 4); it rotates to 15 m_t on
even channels and 0 on odd ones, an exact INT4 group (scale m_t, offset 0),
and loop 0 is exactly 2^26 x, so its LS coefficient is 2^26 and its residual
is zero.  A value weight p * alpha * scale then reaches 2^26 * 1024 = 2^36 for
the token with the largest score.  Batch row 1 holds ordinary Gaussian rows.
The oracle needs none of this: it reconstructs in fp64."""
import numpy as np
import torch

import oracle
import residual_bit_kv_b200.librq as L

B, H, D, T = 2, 1, 64, 96
BITS, GROUP = (2, 4), (32, 32)


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def inputs(seed: int = 11):
    """bf16 bits: xk, xv [loops][B][H][T][D]; q, kcur, vcur [B][H][D]."""
    g = np.random.default_rng(seed)
    xk = np.empty((2, B, H, T, D), np.float32)
    xv = np.empty((2, B, H, T, D), np.float32)
    xk[1] = g.standard_normal((B, H, T, D))
    xk[0] = xk[1] * 1.1 + 0.3 * g.standard_normal((B, H, T, D))
    xv[1, 1] = g.standard_normal((H, T, D))
    xv[0, 1] = xv[1, 1] * 0.9 + 0.3 * g.standard_normal((H, T, D))
    xv[:, 0] = 0.0
    for t in range(T):
        m = 1024.0 * 2.0 ** (t % 4)
        xv[1, 0, :, t, 0:2] = 60.0 * m
    xv[0, 0] = xv[1, 0] * 2.0 ** 26
    q = g.standard_normal((B, H, D))
    kc = g.standard_normal((B, H, D))
    vc = g.standard_normal((B, H, D))
    bits = {k: _bf16(v) for k, v in dict(xk=xk, xv=xv, q=q, kc=kc, vc=vc).items()}
    # the constructed unit is bf16-exact
    assert np.array_equal(((bits["xv"][:, 0].astype(np.uint32) << 16).view(np.float32)), xv[:, 0])
    return bits


def build(bits):
    """Packed cache on the GPU (per-loop appends) and the decode inputs."""
    lay = L.make_layout(1, 2, B, H, D, T, BITS, GROUP, L.RQ_POLICY_LAST_LOOP)
    nb = L.rq_cache_bytes(lay)
    kb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    vb = torch.empty(nb, dtype=torch.uint8, device="cuda")
    cache = L.rq_cache_bind(lay, kb, vb)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        torch.bfloat16).cuda()
    for side, x in ((0, bits["xk"]), (1, bits["xv"])):
        L.rq_quantize_anchor(cache, 0, side, dev(x[1]), 0, T)
        L.rq_quantize_append_residual(cache, 0, side, 0, dev(x[0]), 0, T)
    torch.cuda.synchronize()
    return lay, cache, (kb, vb), dev(bits["q"]), dev(bits["kc"]), dev(bits["vc"])


def oracle_out(bits, b: int, loop: int) -> np.ndarray:
    """fp64 oracle decode of unit (b, 0) for `loop`."""
    rec = {}
    for side, x in ((0, bits["xk"]), (1, bits["xv"])):
        encs = oracle.encode_side(x[:, b, 0], BITS, GROUP)
        rec[side] = oracle.reconstruct(encs, loop, BITS, GROUP)
    f = oracle.bf16_bits_to_f64
    return oracle.attention(f(bits["q"][b, 0]), rec[0], rec[1], f(bits["kc"][b, 0]),
                            f(bits["vc"][b, 0]), 1.0 / np.sqrt(D))
