/*
 * rqo.h -- CPU oracle for the ResidualQuant KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (librq) never calls it and shares no code, header, table or helper with it.
 *
 * Plain, single-threaded, deliberately slow C.  Every function follows one
 * passage of the method's description, cited as
 *   [RQ §x]  = "ResidualQuant: KV Cache Quantization for Looped Transformers
 *              with 2-Bit Residuals" (paperpeel.com/paper/2610.10381), section x.
 *
 * Precision: the quantities that decide an integer (a code, a min/max, the
 * fp16 metadata, the bf16 LS coefficient) are computed in fp32 in one fixed,
 * documented order, so the GPU path can be held to bit-exact agreement.
 * Reconstruction and attention are computed in fp64.
 *
 * Row length: D is a power of two in [32, 256] everywhere (the row
 * functions keep rows in 256-entry stack buffers); the Python wrapper
 * rejects any other D before calling in.
 *
 * Packed formats (the storage contract both sides implement independently):
 *   codes : b = 2: channel i of a row lives in 32-bit word i/16, bits
 *           [2*(i%16), +2).  b = 4: in blocks of 16 channels, i = 16u + v,
 *           word 2u + ((v>>1)&1), bits [4*(2*(v>>2) + (v&1)), +4); this
 *           order puts the same channels in the same byte lanes for both
 *           widths.  Little-endian 32-bit words.
 *   meta  : one 32-bit word per group: low half = fp16 scale s~,
 *           high half = fp16 offset z~.
 *   alpha : bf16 bits of the LS coefficient, one per (token, head).
 */
#ifndef RQO_H
#define RQO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Number conversions, written from the IEEE-754 binary16 / bfloat16
 * definitions (round to nearest, ties to even). */
float    rqo_bf16_to_f32(uint16_t h);
uint16_t rqo_f32_to_bf16(float f);
float    rqo_f16_to_f32(uint16_t h);
uint16_t rqo_f32_to_f16(float f);

/* fp32 normalisation constant of the D x D Sylvester-Hadamard matrix:
 * round-to-nearest fp32 of 1/sqrt(D). */
float rqo_rot_scale(int D);

/* z <- H z, H the normalised Sylvester-Hadamard matrix [RQ §3.3, App. G.2].
 * fp32, stages h = 1, 2, ..., D/2, each pair (a, b) -> (a + b, a - b),
 * then one fp32 multiply by rqo_rot_scale(D). */
void rqo_fwht_f32(float* z, int D);

/* Same transform in fp64, normalised by 1/sqrt(D) in fp64; H = H^T = H^-1. */
void rqo_fwht_f64(double* z, int D);
void rqo_fwht_rows_f64(double* z, int64_t n, int D);

/* Canonical-order fp32 dot product used for the LS coefficient:
 * the D channels are split into P = D/32 consecutive slices of 32; each
 * slice is summed serially with fused multiply-add starting from +0; the P
 * partial sums are then combined by a butterfly: for off = P/2, ..., 1,
 * p[l] <- p[l] + p[l ^ off].  Returns p[0].  Requires D % 32 == 0. */
float rqo_dot_f32(const float* a, const float* b, int D);

/* Word index and bit shift of channel i in a packed row of `bits`-bit codes. */
void rqo_code_pos(int i, int bits, int* word, int* shift);

/* Group-wise affine quantisation of one rotated row [RQ §2.1]:
 * per group of g consecutive channels: mn, mx; s = (mx - mn)/(2^b - 1);
 * s~ = fp16(s), z~ = fp16(mn); inv = 1/s~ (0 if s~ == 0);
 * u = (z - z~) * inv; c = rint_half_even(clamp(u, 0, 2^b - 1));
 * deq = fma(s~, c, z~).  Writes packed words (D*b/32), meta (D/g), deq (D). */
void rqo_quantize(const float* z, int D, int bits, int group,
                  uint32_t* words, uint32_t* meta, float* deq);

/* 16-bit metadata per group (scale byte + offset byte), the storage the
 * pages count for scales and offsets (16 bits per group [RQ §5.1, App. A.3];
 * the pages do not give the format, this one is the library's choice):
 *   scale byte: unsigned e5m3, b = 8 E + m; E = 0 encodes a zero scale,
 *     else s~ = (1 + m/8) * 2^(E - RQO_M8_BIAS), E in 1..31, m in 0..7.
 *   rqo_m8_scale_encode rounds a finite s >= 0 to the nearest such value
 *     (ties to even m), sends s below the smallest positive value to the
 *     smallest and above the largest to the largest; s <= 0 or NaN -> 0. */
#define RQO_M8_BIAS 18
uint8_t rqo_m8_scale_encode(float s);
float   rqo_m8_scale_decode(uint8_t b);

/* Group-wise affine quantisation with 16-bit metadata: per group, mn, mx
 * (+0 for zeros); s0 = (mx - mn)/(2^b - 1); s1 = |mn| / 15.875;
 * s~ = decode(encode(max(s0, s1))) (s1 keeps the offset near the offset
 * byte's range); t = floor((8 mn) / s~); if t is outside [-128, 127] the
 * scale byte is raised by one (next larger value) and t recomputed; offset
 * byte zq = clamp(t, -128, 127) (0 if s~ == 0; the clamp only acts at the
 * largest scale byte), z~ = zq * s~ / 8 (exact); codes and levels as in
 * rqo_quantize: inv = 1/s~ (0 if s~ == 0), c = rint(clamp((z - z~) * inv)),
 * deq = fma(s~, c, z~).  meta[j] = scale byte | (offset byte << 8).
 * Error bound (scales inside the byte's range): s~ is within 1/17 below the
 * range scale and z~ within s~/8 below mn, so every value is within
 * max(1/2, (2^b - 1)/16 + 1/8) * s~ of its level (plus fp32 rounding):
 * half a step for INT2, 1.0625 steps at the top of an INT4 group. */
void rqo_quantize_m8(const float* z, int D, int bits, int group,
                     uint32_t* words, uint16_t* meta, float* deq);

/* Anchor of the final loop [RQ §3.2 Last-loop policy, §3.4, App. G.2]:
 * Z = H x (x bf16), quantised with the anchor's bits and group.
 * zhat receives the dequantised rotated anchor A (fp32). */
void rqo_encode_anchor(const uint16_t* x, int D, int bits, int group,
                       uint32_t* words, uint32_t* meta, float* zhat);

/* Residual loop from an already rotated fp32 row z and reference ref
 * (rotated, dequantised) [RQ §3.2 scaling coefficient, App. G.1]:
 * alpha = <z, ref>/<ref, ref> (0 when <ref, ref> == 0), both dots by
 * rqo_dot_f32, one IEEE division; alpha~ = bf16(alpha);
 * E = fma(-alpha~, ref, z); E quantised with (bits, group);
 * zhat = fma(alpha~, ref, deq(E)) is the reconstructed rotated row. */
void rqo_encode_residual_rot(const float* z, const float* ref, int D, int bits,
                             int group, int unit_alpha, uint32_t* words,
                             uint32_t* meta, uint16_t* alpha, float* zhat);

/* Same, from a bf16 row x (rotated here with rqo_fwht_f32). */
void rqo_encode_residual(const uint16_t* x, const float* ref, int D, int bits,
                         int group, int unit_alpha, uint32_t* words,
                         uint32_t* meta, uint16_t* alpha, float* zhat);

/* Row-batched forms of the two encoders: n rows, row-major. */
void rqo_encode_anchor_rows(const uint16_t* x, int64_t n, int D, int bits,
                            int group, uint32_t* words, uint32_t* meta,
                            float* zhat);
void rqo_encode_residual_rows(const uint16_t* x, const float* ref, int64_t n,
                              int D, int bits, int group, int unit_alpha,
                              uint32_t* words, uint32_t* meta, uint16_t* alpha,
                              float* zhat);

/* fp64 value of the stored levels of one packed row: s~ * c + z~. */
void rqo_dequant_codes_f64(const uint32_t* words, const uint32_t* meta, int D,
                           int bits, int group, double* out);
void rqo_dequant_rows_f64(const uint32_t* words, const uint32_t* meta,
                          int64_t n, int D, int bits, int group, double* out);

/* The encoders, the row forms and the level reconstruction with 16-bit
 * metadata (rqo_quantize_m8 in place of rqo_quantize; meta uint16 per
 * group); every other step as in the functions above. */
void rqo_encode_anchor_rows_m8(const uint16_t* x, int64_t n, int D, int bits,
                               int group, uint32_t* words, uint16_t* meta,
                               float* zhat);
void rqo_encode_residual_rot_m8(const float* z, const float* ref, int D, int bits,
                                int group, int unit_alpha, uint32_t* words,
                                uint16_t* meta, uint16_t* alpha, float* zhat);
void rqo_encode_residual_rows_m8(const uint16_t* x, const float* ref, int64_t n,
                                 int D, int bits, int group, int unit_alpha,
                                 uint32_t* words, uint16_t* meta,
                                 uint16_t* alpha, float* zhat);
void rqo_dequant_rows_m8_f64(const uint32_t* words, const uint16_t* meta,
                             int64_t n, int D, int bits, int group, double* out);

/* Residual encoder with a fixed mean [RQ App. G.2: Z^_r = alpha_r A +
 * D(c_r) + mu_r] and either metadata form: zc = z - mu (mu NULL: no mean);
 * alpha = <zc, ref>/<ref, ref> (1 with unit_alpha); E = fma(-alpha~, ref, zc)
 * quantised with rqo_quantize (meta uint32) or rqo_quantize_m8 (meta16:
 * meta uint16); zhat = fma(alpha~, ref, deq(E)) + mu.  Row forms take x
 * (bf16, rotated here), ref and mu as n rows of D. */
void rqo_encode_residual_rot_ex(const float* z, const float* ref, const float* mu,
                                int D, int bits, int group, int unit_alpha,
                                int meta16, uint32_t* words, void* meta,
                                uint16_t* alpha, float* zhat);
void rqo_encode_residual_rows_ex(const uint16_t* x, const float* ref,
                                 const float* mu, int64_t n, int D, int bits,
                                 int group, int unit_alpha, int meta16,
                                 uint32_t* words, void* meta, uint16_t* alpha,
                                 float* zhat);

/* Softmax attention of one query against T rows, fp64 [RQ §4.1, §4.2,
 * App. G.1]: s_t = scale * q.k_t for t < T, plus the current token
 * s_cur = scale * q.k_cur; p = softmax(s); out = sum_t p_t v_t + p_cur v_cur.
 * khat and vhat are T x D row-major (original domain). */
/* Dense rotation [RQ §3.3, App. G.2]: z = U x with U binary16 (row i =
 * output channel i) and x rounded from bf16 to binary16; z in fp64 and, per
 * channel, a bound on the error of any order of fp32 accumulation. */
void rqo_rotate_dense_row(const uint16_t* u, const uint16_t* x, int D, double* z,
                          double* bound);
void rqo_rotate_dense_rows(const uint16_t* u, const uint16_t* x, int64_t n, int D,
                           double* z, double* bound);
/* Interval forms of the quantiser and of the residual encoder (binary16
 * metadata): the decisions shared by every row of the box [lo, hi]. */
void rqo_quantize_box(const float* lo, const float* hi, const float* mid, int D,
                      int bits, int group, uint32_t* words, uint32_t* meta, float* deq,
                      uint8_t* meta_ok, uint8_t* code_ok);
void rqo_encode_residual_box(const float* lo, const float* hi, const float* mid,
                             const float* ref, const float* mu, int D, int bits, int group,
                             int unit_alpha, uint32_t* words, uint32_t* meta,
                             uint16_t* alpha, float* zhat, uint8_t* alpha_ok,
                             uint8_t* meta_ok, uint8_t* code_ok);

void rqo_quantize_box_rows(const float* lo, const float* hi, const float* mid, int64_t n,
                           int D, int bits, int group, uint32_t* words, uint32_t* meta,
                           float* deq, uint8_t* meta_ok, uint8_t* code_ok);
void rqo_encode_residual_box_rows(const float* lo, const float* hi, const float* mid,
                                  const float* ref, const float* mu, int64_t n, int D,
                                  int bits, int group, int unit_alpha, uint32_t* words,
                                  uint32_t* meta, uint16_t* alpha, float* zhat,
                                  uint8_t* alpha_ok, uint8_t* meta_ok, uint8_t* code_ok);

void rqo_attention_f64(const double* q, const double* khat, const double* vhat,
                       int64_t T, const double* kcur, const double* vcur,
                       int D, double scale, double* out);

/* Effective bits per KV element [RQ App. A.3]: codes, scales, offsets and LS
 * coefficients, averaged over the L loops of a group.  bits[r], group[r] for
 * r = 0..L-1 (loop L-1 is the anchor); meta_bits = bits of (scale + offset)
 * per group; residual != 0 adds one 16-bit coefficient per (token, head) for
 * each of the L-1 non-anchor loops. */
double rqo_effective_bits(int L, const int* bits, const int* group, int D,
                          int meta_bits, int residual);

/* Logical compressed-component reads needed to reconstruct every loop of a
 * group of L loops [RQ App. D, logical reference count]:
 * shared anchor (First-/Last-loop): 2L - 1; chained (Previous-/Next-loop):
 * L(L+1)/2.  chained selects the policy. */
int64_t rqo_component_reads(int L, int chained);

#ifdef __cplusplus
}
#endif

#endif /* RQO_H */
