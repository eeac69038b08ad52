/*
 * rqo.c -- CPU oracle for the ResidualQuant KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see rqo.h).  Plain scalar loops, one row at a
 * time, in the order the method states them.  Build with
 *   gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * so that no multiply-add is fused except the explicit fmaf() calls.
 *
 * Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
 * Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
 */
#include "rqo.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

float rqo_bf16_to_f32(uint16_t h) {
  /* bfloat16 is the upper half of an IEEE binary32. */
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

uint16_t rqo_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays NaN */
  /* Drop the low 16 bits, rounding to nearest with ties to even. */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

float rqo_f16_to_f32(uint16_t h) {
  /* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
  int sign = h >> 15;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  float v;
  if (e == 0)
    v = ldexpf((float)m, -24);                 /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexpf((float)(m + 1024), e - 25);     /* (1 + m/1024) * 2^(e-15) */
  return sign ? -v : v;
}

uint16_t rqo_f32_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  float a = fabsf(f);
  if (isnan(a)) return sign | 0x7E00u;
  if (isinf(a)) return sign | 0x7C00u;
  if (a < 0x1p-14f) {
    /* Subnormal range: the unit in the last place is 2^-24.  a * 2^24 is an
     * exact power-of-two scaling; rintf rounds half to even.  A result of
     * 1024 is exactly the encoding of the smallest normal, 2^-14. */
    float m = rintf(a * 0x1p24f);
    return sign | (uint16_t)m;
  }
  int e;
  (void)frexpf(a, &e);       /* a in [2^(e-1), 2^e) */
  e -= 1;                    /* a in [2^e, 2^(e+1)), ulp = 2^(e-10) */
  float m = rintf(ldexpf(a, 10 - e));   /* in [1024, 2048] */
  if (m == 2048.0f) {
    m = 1024.0f;
    e += 1;
  }
  if (e > 15) return sign | 0x7C00u;   /* overflow rounds to infinity */
  return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0f);
}

/* ------------------------------------------------------------------------ */
/* Rotation: normalised Sylvester-Hadamard [RQ §3.3, App. G.1, App. G.2]     */
/* ------------------------------------------------------------------------ */

float rqo_rot_scale(int D) { return (float)(1.0 / sqrt((double)D)); }

void rqo_fwht_f32(float* z, int D) {
  for (int h = 1; h < D; h *= 2)
    for (int i = 0; i < D; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        float a = z[j], b = z[j + h];
        z[j] = a + b;
        z[j + h] = a - b;
      }
  const float c = rqo_rot_scale(D);
  for (int i = 0; i < D; ++i) z[i] = z[i] * c;
}

void rqo_fwht_f64(double* z, int D) {
  for (int h = 1; h < D; h *= 2)
    for (int i = 0; i < D; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        double a = z[j], b = z[j + h];
        z[j] = a + b;
        z[j + h] = a - b;
      }
  const double c = 1.0 / sqrt((double)D);
  for (int i = 0; i < D; ++i) z[i] *= c;
}

void rqo_fwht_rows_f64(double* z, int64_t n, int D) {
  for (int64_t r = 0; r < n; ++r) rqo_fwht_f64(z + r * D, D);
}

/* ------------------------------------------------------------------------ */
/* LS coefficient dot product in its canonical order                        */
/* ------------------------------------------------------------------------ */

float rqo_dot_f32(const float* a, const float* b, int D) {
  float p[8];
  const int P = D / 32;
  for (int l = 0; l < P; ++l) {
    float acc = 0.0f;
    for (int k = 0; k < 32; ++k) acc = fmaf(a[32 * l + k], b[32 * l + k], acc);
    p[l] = acc;
  }
  for (int off = P / 2; off >= 1; off /= 2) {
    float q[8];
    for (int l = 0; l < P; ++l) q[l] = p[l] + p[l ^ off];
    for (int l = 0; l < P; ++l) p[l] = q[l];
  }
  return p[0];
}

/* ------------------------------------------------------------------------ */
/* Group-wise affine quantisation [RQ §2.1]                                  */
/* ------------------------------------------------------------------------ */

/* Storage position of channel i of a row (word index, bit shift).
 * b = 2: word i/16, bits 2*(i%16).
 * b = 4: channels come in blocks of 16 (i = 16u + v); word 2u + ((v>>1)&1),
 *        nibble 2*(v>>2) + (v&1), i.e. bits 4*nibble. */
void rqo_code_pos(int i, int bits, int* word, int* shift) {
  if (bits == 2) {
    *word = i / 16;
    *shift = 2 * (i % 16);
  } else {
    const int u = i / 16, v = i % 16;
    *word = 2 * u + ((v >> 1) & 1);
    *shift = 4 * (2 * (v >> 2) + (v & 1));
  }
}

void rqo_quantize(const float* z, int D, int bits, int group, uint32_t* words,
                  uint32_t* meta, float* deq) {
  const int qmax = (1 << bits) - 1;
  for (int w = 0; w < D * bits / 32; ++w) words[w] = 0u;

  for (int g0 = 0, j = 0; g0 < D; g0 += group, ++j) {
    /* Range of the group. */
    float mn = z[g0], mx = z[g0];
    for (int i = g0 + 1; i < g0 + group; ++i) {
      if (z[i] < mn) mn = z[i];
      if (z[i] > mx) mx = z[i];
    }
    mn = mn + 0.0f; /* a zero range end is taken as +0 */
    mx = mx + 0.0f;

    /* Scale and offset, stored as fp16; levels are z~ + k s~, k = 0..qmax. */
    const float s = (mx - mn) / (float)qmax;
    const uint16_t sh = rqo_f32_to_f16(s);
    const uint16_t zh = rqo_f32_to_f16(mn);
    const float st = rqo_f16_to_f32(sh);
    const float zt = rqo_f16_to_f32(zh);
    const float inv = (st > 0.0f) ? 1.0f / st : 0.0f;
    meta[j] = (uint32_t)sh | ((uint32_t)zh << 16);

    /* Nearest level: round half to even, clamped to the code range. */
    for (int i = g0; i < g0 + group; ++i) {
      float u = (z[i] - zt) * inv;
      if (u < 0.0f) u = 0.0f;
      if (u > (float)qmax) u = (float)qmax;
      const uint32_t code = (uint32_t)rintf(u);
      int wi, bit;
      rqo_code_pos(i, bits, &wi, &bit);
      words[wi] |= code << bit;
      deq[i] = fmaf(st, (float)code, zt);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 16-bit metadata variant [RQ §5.1, App. A.3: 16 bits of scale and offset  */
/* per group]                                                              */
/* ------------------------------------------------------------------------ */

uint8_t rqo_m8_scale_encode(float s) {
  if (!(s > 0.0f)) return 0u;                       /* zero, negative, NaN */
  uint32_t b;
  memcpy(&b, &s, sizeof(b));
  int E = (int)((b >> 23) & 0xFFu);
  if (E == 0xFF) return 0xFFu;                      /* infinity: the largest */
  if (E == 0) return 0x08u;                         /* fp32 subnormal: the smallest */
  uint32_t m = (b & 0x7FFFFFu) >> 20;               /* top 3 mantissa bits */
  const uint32_t rem = b & 0xFFFFFu;                /* the 20 bits dropped */
  if (rem > 0x80000u || (rem == 0x80000u && (m & 1u))) ++m;
  if (m == 8u) {
    m = 0u;
    ++E;
  }
  const int Eb = E - 127 + RQO_M8_BIAS;
  if (Eb < 1) return 0x08u;
  if (Eb > 31) return 0xFFu;
  return (uint8_t)(((uint32_t)Eb << 3) | m);
}

float rqo_m8_scale_decode(uint8_t b) {
  const int Eb = b >> 3, m = b & 7;
  if (Eb == 0) return 0.0f;
  return ldexpf(1.0f + (float)m / 8.0f, Eb - RQO_M8_BIAS);
}

void rqo_quantize_m8(const float* z, int D, int bits, int group, uint32_t* words,
                     uint16_t* meta, float* deq) {
  const int qmax = (1 << bits) - 1;
  for (int w = 0; w < D * bits / 32; ++w) words[w] = 0u;

  for (int g0 = 0, j = 0; g0 < D; g0 += group, ++j) {
    float mn = z[g0], mx = z[g0];
    for (int i = g0 + 1; i < g0 + group; ++i) {
      if (z[i] < mn) mn = z[i];
      if (z[i] > mx) mx = z[i];
    }
    mn = mn + 0.0f;
    mx = mx + 0.0f;

    /* Scale: the range over the code steps, at least |mn| / 15.875 so that
     * the offset fits its byte; rounded to the scale byte. */
    const float s0 = (mx - mn) / (float)qmax;
    const float s1 = fabsf(mn) / 15.875f;
    uint8_t sb = rqo_m8_scale_encode(s0 > s1 ? s0 : s1);
    float st = rqo_m8_scale_decode(sb);

    /* Offset: the largest multiple of s~/8 not above mn.  When the nearest
     * scale rounded down far enough that this multiple leaves the offset
     * byte, the scale byte goes up one step (one step always suffices); the
     * clamp is left only for the largest scale byte. */
    int zq = 0;
    if (st > 0.0f) {
      float t = floorf((8.0f * mn) / st);
      if ((t < -128.0f || t > 127.0f) && sb < 0xFFu) {
        sb = (uint8_t)(sb + 1u);
        st = rqo_m8_scale_decode(sb);
        t = floorf((8.0f * mn) / st);
      }
      zq = t < -128.0f ? -128 : (t > 127.0f ? 127 : (int)t);
    }
    const float zt = (float)zq * st * 0.125f;
    const float inv = (st > 0.0f) ? 1.0f / st : 0.0f;
    meta[j] = (uint16_t)((uint32_t)sb | (((uint32_t)zq & 0xFFu) << 8));

    for (int i = g0; i < g0 + group; ++i) {
      float u = (z[i] - zt) * inv;
      if (u < 0.0f) u = 0.0f;
      if (u > (float)qmax) u = (float)qmax;
      const uint32_t code = (uint32_t)rintf(u);
      int wi, bit;
      rqo_code_pos(i, bits, &wi, &bit);
      words[wi] |= code << bit;
      deq[i] = fmaf(st, (float)code, zt);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Anchor and residual encoders [RQ §3.2, §3.3, §3.4, App. G.1, App. G.2]    */
/* ------------------------------------------------------------------------ */

void rqo_encode_anchor(const uint16_t* x, int D, int bits, int group,
                       uint32_t* words, uint32_t* meta, float* zhat) {
  float z[256];
  for (int i = 0; i < D; ++i) z[i] = rqo_bf16_to_f32(x[i]);
  rqo_fwht_f32(z, D);
  rqo_quantize(z, D, bits, group, words, meta, zhat);
}

void rqo_encode_residual_rot(const float* z, const float* ref, int D, int bits,
                             int group, int unit_alpha, uint32_t* words,
                             uint32_t* meta, uint16_t* alpha, float* zhat) {
  /* Least-squares scale of the reference: alpha = <X_r, R>/||R||^2 [RQ §3.2
   * scaling coefficient]; alpha = 1 without LS scaling (the plain
   * inter-loop difference of the Previous-loop description, and the "w/o LS
   * scaling" columns of [RQ Table 3]). */
  float a = 1.0f;
  if (!unit_alpha) {
    const float d_zr = rqo_dot_f32(z, ref, D);
    const float d_rr = rqo_dot_f32(ref, ref, D);
    a = (d_rr > 0.0f) ? d_zr / d_rr : 0.0f;
  }
  const uint16_t ab = rqo_f32_to_bf16(a);
  const float at = rqo_bf16_to_f32(ab);
  *alpha = ab;

  /* Residual against the stored (bf16) coefficient, then affine quantise. */
  float e[256], deq[256];
  for (int i = 0; i < D; ++i) e[i] = fmaf(-at, ref[i], z[i]);
  rqo_quantize(e, D, bits, group, words, meta, deq);

  /* Reconstructed rotated row (the reference of a chained predecessor). */
  for (int i = 0; i < D; ++i) zhat[i] = fmaf(at, ref[i], deq[i]);
}

void rqo_encode_residual(const uint16_t* x, const float* ref, int D, int bits,
                         int group, int unit_alpha, uint32_t* words,
                         uint32_t* meta, uint16_t* alpha, float* zhat) {
  float z[256];
  for (int i = 0; i < D; ++i) z[i] = rqo_bf16_to_f32(x[i]);
  rqo_fwht_f32(z, D);
  rqo_encode_residual_rot(z, ref, D, bits, group, unit_alpha, words, meta, alpha,
                          zhat);
}

void rqo_encode_anchor_rows(const uint16_t* x, int64_t n, int D, int bits,
                            int group, uint32_t* words, uint32_t* meta,
                            float* zhat) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r)
    rqo_encode_anchor(x + r * D, D, bits, group, words + r * W, meta + r * G,
                      zhat + r * D);
}

void rqo_encode_residual_rows(const uint16_t* x, const float* ref, int64_t n,
                              int D, int bits, int group, int unit_alpha,
                              uint32_t* words, uint32_t* meta, uint16_t* alpha,
                              float* zhat) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r)
    rqo_encode_residual(x + r * D, ref + r * D, D, bits, group, unit_alpha,
                        words + r * W, meta + r * G, alpha + r, zhat + r * D);
}

/* ------------------------------------------------------------------------ */
/* Reconstruction and attention in fp64 [RQ §4.1, App. G.2]                  */
/* ------------------------------------------------------------------------ */

void rqo_dequant_codes_f64(const uint32_t* words, const uint32_t* meta, int D,
                           int bits, int group, double* out) {
  const uint32_t qmax = (1u << bits) - 1u;
  for (int i = 0; i < D; ++i) {
    int wi, sh;
    rqo_code_pos(i, bits, &wi, &sh);
    const uint32_t code = (words[wi] >> sh) & qmax;
    const uint32_t m = meta[i / group];
    const double s = rqo_f16_to_f32((uint16_t)(m & 0xFFFFu));
    const double z = rqo_f16_to_f32((uint16_t)(m >> 16));
    out[i] = s * (double)code + z;
  }
}

void rqo_dequant_rows_f64(const uint32_t* words, const uint32_t* meta,
                          int64_t n, int D, int bits, int group, double* out) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r)
    rqo_dequant_codes_f64(words + r * W, meta + r * G, D, bits, group,
                          out + r * D);
}

/* ------------------------------------------------------------------------ */
/* Encoders and levels with 16-bit metadata                                  */
/* ------------------------------------------------------------------------ */

void rqo_encode_anchor_rows_m8(const uint16_t* x, int64_t n, int D, int bits,
                               int group, uint32_t* words, uint16_t* meta,
                               float* zhat) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r) {
    float z[256];
    for (int i = 0; i < D; ++i) z[i] = rqo_bf16_to_f32(x[r * D + i]);
    rqo_fwht_f32(z, D);
    rqo_quantize_m8(z, D, bits, group, words + r * W, meta + r * G, zhat + r * D);
  }
}

void rqo_encode_residual_rot_m8(const float* z, const float* ref, int D, int bits,
                                int group, int unit_alpha, uint32_t* words,
                                uint16_t* meta, uint16_t* alpha, float* zhat) {
  float a = 1.0f;
  if (!unit_alpha) {
    const float d_zr = rqo_dot_f32(z, ref, D);
    const float d_rr = rqo_dot_f32(ref, ref, D);
    a = (d_rr > 0.0f) ? d_zr / d_rr : 0.0f;
  }
  const uint16_t ab = rqo_f32_to_bf16(a);
  const float at = rqo_bf16_to_f32(ab);
  *alpha = ab;
  float e[256], deq[256];
  for (int i = 0; i < D; ++i) e[i] = fmaf(-at, ref[i], z[i]);
  rqo_quantize_m8(e, D, bits, group, words, meta, deq);
  for (int i = 0; i < D; ++i) zhat[i] = fmaf(at, ref[i], deq[i]);
}

void rqo_encode_residual_rows_m8(const uint16_t* x, const float* ref, int64_t n,
                                 int D, int bits, int group, int unit_alpha,
                                 uint32_t* words, uint16_t* meta,
                                 uint16_t* alpha, float* zhat) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r) {
    float z[256];
    for (int i = 0; i < D; ++i) z[i] = rqo_bf16_to_f32(x[r * D + i]);
    rqo_fwht_f32(z, D);
    rqo_encode_residual_rot_m8(z, ref + r * D, D, bits, group, unit_alpha,
                               words + r * W, meta + r * G, alpha + r, zhat + r * D);
  }
}

void rqo_dequant_rows_m8_f64(const uint32_t* words, const uint16_t* meta,
                             int64_t n, int D, int bits, int group, double* out) {
  const int W = D * bits / 32, G = D / group;
  const uint32_t qmax = (1u << bits) - 1u;
  for (int64_t r = 0; r < n; ++r)
    for (int i = 0; i < D; ++i) {
      int wi, sh;
      rqo_code_pos(i, bits, &wi, &sh);
      const uint32_t code = (words[r * W + wi] >> sh) & qmax;
      const uint16_t m = meta[r * G + i / group];
      const double st = rqo_m8_scale_decode((uint8_t)(m & 0xFFu));
      const double zt = (double)(int8_t)(uint8_t)(m >> 8) * st * 0.125;
      out[r * D + i] = st * (double)code + zt;
    }
}

/* ------------------------------------------------------------------------ */
/* Residual encoder with a fixed mean [RQ App. G.2]                          */
/* ------------------------------------------------------------------------ */

void rqo_encode_residual_rot_ex(const float* z, const float* ref, const float* mu,
                                int D, int bits, int group, int unit_alpha,
                                int meta16, uint32_t* words, void* meta,
                                uint16_t* alpha, float* zhat) {
  float zc[256], e[256], deq[256];
  for (int i = 0; i < D; ++i) zc[i] = mu ? z[i] - mu[i] : z[i];
  float a = 1.0f;
  if (!unit_alpha) {
    const float d_zr = rqo_dot_f32(zc, ref, D);
    const float d_rr = rqo_dot_f32(ref, ref, D);
    a = (d_rr > 0.0f) ? d_zr / d_rr : 0.0f;
  }
  const uint16_t ab = rqo_f32_to_bf16(a);
  const float at = rqo_bf16_to_f32(ab);
  *alpha = ab;
  for (int i = 0; i < D; ++i) e[i] = fmaf(-at, ref[i], zc[i]);
  if (meta16)
    rqo_quantize_m8(e, D, bits, group, words, (uint16_t*)meta, deq);
  else
    rqo_quantize(e, D, bits, group, words, (uint32_t*)meta, deq);
  for (int i = 0; i < D; ++i) {
    const float r = fmaf(at, ref[i], deq[i]);
    zhat[i] = mu ? r + mu[i] : r;
  }
}

void rqo_encode_residual_rows_ex(const uint16_t* x, const float* ref,
                                 const float* mu, int64_t n, int D, int bits,
                                 int group, int unit_alpha, int meta16,
                                 uint32_t* words, void* meta, uint16_t* alpha,
                                 float* zhat) {
  const int W = D * bits / 32, G = D / group;
  const size_t mb = meta16 ? 2 : 4;
  for (int64_t r = 0; r < n; ++r) {
    float z[256];
    for (int i = 0; i < D; ++i) z[i] = rqo_bf16_to_f32(x[r * D + i]);
    rqo_fwht_f32(z, D);
    rqo_encode_residual_rot_ex(z, ref + r * D, mu ? mu + r * D : NULL, D, bits, group,
                               unit_alpha, meta16, words + r * W,
                               (unsigned char*)meta + (size_t)(r * G) * mb, alpha + r,
                               zhat + r * D);
  }
}

void rqo_attention_f64(const double* q, const double* khat, const double* vhat,
                       int64_t T, const double* kcur, const double* vcur, int D,
                       double scale, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(T + 1));
  double m;
  {
    double d = 0.0;
    for (int i = 0; i < D; ++i) d += q[i] * kcur[i];
    s[T] = scale * d;
    m = s[T];
  }
  for (int64_t t = 0; t < T; ++t) {
    double d = 0.0;
    for (int i = 0; i < D; ++i) d += q[i] * khat[t * D + i];
    s[t] = scale * d;
    if (s[t] > m) m = s[t];
  }
  double l = exp(s[T] - m);
  for (int i = 0; i < D; ++i) out[i] = l * vcur[i];
  for (int64_t t = 0; t < T; ++t) {
    const double p = exp(s[t] - m);
    l += p;
    for (int i = 0; i < D; ++i) out[i] += p * vhat[t * D + i];
  }
  for (int i = 0; i < D; ++i) out[i] /= l;
  free(s);
}

/* ------------------------------------------------------------------------ */
/* Dense rotation [RQ §3.3, App. G.1, App. G.2]                              */
/* ------------------------------------------------------------------------ */

/* z = U x for one row.  U is D x D in binary16, row i giving output channel
 * i; x is the bf16 row rounded to binary16 (the pages: rotation matrices
 * stored in FP16, multiplication with FP16 inputs and FP32 accumulation).
 * A product of two binary16 values is exact in binary32 and in fp64.  The
 * pages fix the accumulator's precision but not the order of its D
 * additions, so the oracle returns the sum formed in fp64 together with a
 * bound that every order of fp32 accumulation of the exact products meets:
 *   bound_i = D 2^-23 sum_j |U_ij x_j|  (+ the fp64 sum's own D 2^-53 share),
 * twice the textbook (D - 1) 2^-24, which also covers adders that truncate;
 * the bound is 0 when every partial sum is exact in any order (below). */
/* Exponent of the lowest set bit of a nonzero binary16 value (from its bits):
 * a normal value is (1024 + m) 2^(e - 25), a subnormal one m 2^-24. */
static int f16_low_bit(uint16_t h) {
  const int e = (h >> 10) & 0x1F, m = h & 0x3FF;
  return e == 0 ? -24 + __builtin_ctz((unsigned)m) : e - 25 + __builtin_ctz((unsigned)(m | 1024));
}

/* One row against a matrix already decoded: ud[i*D + j] = U_ij as a double,
 * ulow[i*D + j] = the exponent of its lowest set bit. */
static void rotate_dense_decoded(const double* ud, const int* ulow, const uint16_t* x, int D,
                                 double* z, double* bound) {
  double xh[256];
  int xlow[256];
  for (int j = 0; j < D; ++j) {
    const uint16_t hb = rqo_f32_to_f16(rqo_bf16_to_f32(x[j]));
    xh[j] = rqo_f16_to_f32(hb);
    xlow[j] = (hb & 0x7FFF) ? f16_low_bit(hb) : 0;
  }
  for (int i = 0; i < D; ++i) {
    double acc = 0.0, mag = 0.0;
    int emin = 1 << 20;
    for (int j = 0; j < D; ++j) {
      const double t = ud[(size_t)i * D + j] * xh[j];
      acc += t;
      mag += fabs(t);
      if (t != 0.0) {   /* the product's lowest bit: the sum of its factors' */
        const int e = ulow[(size_t)i * D + j] + xlow[j];
        if (e < emin) emin = e;
      }
    }
    z[i] = acc;
    /* Every term a multiple of 2^emin and sum |t| < 2^(24 + emin): each partial
     * sum of any subset, in any order, is such a multiple below 2^(24 + emin),
     * exact in fp32 (and in fp64): no rounding anywhere. */
    if (mag == 0.0 || mag < ldexp(1.0, 24 + emin))
      bound[i] = 0.0;
    else
      bound[i] = mag * ((double)D * 0x1p-23 + (double)D * 0x1p-53);
  }
}

static void decode_matrix(const uint16_t* u, int D, double* ud, int* ulow) {
  for (int k = 0; k < D * D; ++k) {
    ud[k] = rqo_f16_to_f32(u[k]);
    ulow[k] = (u[k] & 0x7FFF) ? f16_low_bit(u[k]) : 0;
  }
}

void rqo_rotate_dense_row(const uint16_t* u, const uint16_t* x, int D, double* z,
                          double* bound) {
  rqo_rotate_dense_rows(u, x, 1, D, z, bound);
}

void rqo_rotate_dense_rows(const uint16_t* u, const uint16_t* x, int64_t n, int D,
                           double* z, double* bound) {
  double* ud = (double*)malloc(sizeof(double) * (size_t)D * D);
  int* ulow = (int*)malloc(sizeof(int) * (size_t)D * D);
  decode_matrix(u, D, ud, ulow);
  for (int64_t r = 0; r < n; ++r)
    rotate_dense_decoded(ud, ulow, x + r * D, D, z + r * D, bound + r * D);
  free(ud);
  free(ulow);
}

/* Interval form of rqo_quantize for a row known only to lie in the box
 * [lo_i, hi_i]: which decisions every row of the box shares.  Each step is
 * monotone in its inputs: the group min and max are non-decreasing in every
 * element, the fp32 scale (mx - mn) / qmax is non-decreasing in mx and
 * non-increasing in mn, binary16 rounding, the code's fsub / fmul by a
 * non-negative inverse, the clamp and rint are non-decreasing.  So the
 * group's metadata is the same for the whole box (meta_ok) when the ends of
 * the offset's and the scale's intervals round to the same binary16 value,
 * and a channel's code is the same (code_ok) when, besides, both ends of its
 * own interval give the same code.  words / meta / deq are those of mid. */
void rqo_quantize_box(const float* lo, const float* hi, const float* mid, int D,
                      int bits, int group, uint32_t* words, uint32_t* meta, float* deq,
                      uint8_t* meta_ok, uint8_t* code_ok) {
  const int qmax = (1 << bits) - 1;
  rqo_quantize(mid, D, bits, group, words, meta, deq);
  for (int g0 = 0, j = 0; g0 < D; g0 += group, ++j) {
    float mn_lo = lo[g0], mn_hi = hi[g0], mx_lo = lo[g0], mx_hi = hi[g0];
    for (int i = g0 + 1; i < g0 + group; ++i) {
      if (lo[i] < mn_lo) mn_lo = lo[i];
      if (hi[i] < mn_hi) mn_hi = hi[i];
      if (lo[i] > mx_lo) mx_lo = lo[i];
      if (hi[i] > mx_hi) mx_hi = hi[i];
    }
    mn_lo = mn_lo + 0.0f;
    mn_hi = mn_hi + 0.0f;
    mx_lo = mx_lo + 0.0f;
    mx_hi = mx_hi + 0.0f;
    const float s_lo = (mx_lo - mn_hi) / (float)qmax;
    const float s_hi = (mx_hi - mn_lo) / (float)qmax;
    const int ok = rqo_f32_to_f16(mn_lo) == rqo_f32_to_f16(mn_hi) &&
                   rqo_f32_to_f16(s_lo) == rqo_f32_to_f16(s_hi);
    meta_ok[j] = (uint8_t)ok;
    const float st = rqo_f16_to_f32((uint16_t)(meta[j] & 0xFFFFu));
    const float zt = rqo_f16_to_f32((uint16_t)(meta[j] >> 16));
    const float inv = (st > 0.0f) ? 1.0f / st : 0.0f;
    for (int i = g0; i < g0 + group; ++i) {
      float ua = (lo[i] - zt) * inv, ub = (hi[i] - zt) * inv;
      if (ua < 0.0f) ua = 0.0f;
      if (ua > (float)qmax) ua = (float)qmax;
      if (ub < 0.0f) ub = 0.0f;
      if (ub > (float)qmax) ub = (float)qmax;
      code_ok[i] = (uint8_t)(ok && rintf(ua) == rintf(ub));
    }
  }
}

/* Interval form of the residual encoder (rqo_encode_residual_rot_ex with
 * binary16 metadata) for a row z in the box [lo, hi] and an exactly known
 * reference (and mean).  The mean's fsub is non-decreasing in z.  Any row of
 * the box has a lane-serial fp32 dot <z - mu, ref> within
 *   sum_i |ref_i| (hi_i - lo_i) + 35 2^-24 sum_i (|mid_i - mu_i| + hi_i - lo_i) |ref_i|
 * of the fp64 dot of mid (32 serial fma roundings and at most 3 butterfly
 * additions, each within 2^-24 of its partial sum); d_zr / d_rr is monotone
 * in d_zr (d_rr > 0 is the same fp32 value for every row: ref is known), so
 * alpha~ is the same for the whole box (alpha_ok) when bf16 rounding maps
 * the quotients of the ends of that interval to one value.  With alpha~
 * fixed the residual fma(-alpha~, ref_i, z_i) is non-decreasing in z_i and its
 * box is the image of the ends; rqo_quantize_box takes it from there.
 * With alpha~ not unique every flag of the row is cleared. */
void rqo_encode_residual_box(const float* lo, const float* hi, const float* mid,
                             const float* ref, const float* mu, int D, int bits, int group,
                             int unit_alpha, uint32_t* words, uint32_t* meta,
                             uint16_t* alpha, float* zhat, uint8_t* alpha_ok,
                             uint8_t* meta_ok, uint8_t* code_ok) {
  rqo_encode_residual_rot_ex(mid, ref, mu, D, bits, group, unit_alpha, 0, words, meta, alpha,
                             zhat);
  const float at = rqo_bf16_to_f32(*alpha);
  int aok = 1;
  if (!unit_alpha) {
    const float d_rr = rqo_dot_f32(ref, ref, D);
    if (d_rr > 0.0f) {
      double c = 0.0, w = 0.0, m = 0.0;
      for (int i = 0; i < D; ++i) {
        const double zc = mu ? (double)mid[i] - (double)mu[i] : (double)mid[i];
        const double wd = (double)hi[i] - (double)lo[i];
        c += zc * (double)ref[i];
        w += fabs((double)ref[i]) * wd;
        m += (fabs(zc) + wd) * fabs((double)ref[i]);
      }
      /* A box of zero width holds one row, whose fp32 dot is the oracle's own;
       * otherwise the fp32 values bracketing every attainable d_zr. */
      if (w > 0.0) {
        const double dev = w + 35.0 * 0x1p-24 * m + (double)D * 0x1p-52 * m;
        const float dlo = nextafterf((float)(c - dev), -INFINITY);
        const float dhi = nextafterf((float)(c + dev), INFINITY);
        aok = rqo_f32_to_bf16(dlo / d_rr) == rqo_f32_to_bf16(dhi / d_rr);
      }
    }
  }
  *alpha_ok = (uint8_t)aok;
  float elo[256], ehi[256], emid[256], deq[256];
  uint32_t w2[64], m2[256];
  for (int i = 0; i < D; ++i) {
    const float zl = mu ? lo[i] - mu[i] : lo[i];
    const float zh = mu ? hi[i] - mu[i] : hi[i];
    const float zm = mu ? mid[i] - mu[i] : mid[i];
    elo[i] = fmaf(-at, ref[i], zl);
    ehi[i] = fmaf(-at, ref[i], zh);
    emid[i] = fmaf(-at, ref[i], zm);
  }
  rqo_quantize_box(elo, ehi, emid, D, bits, group, w2, m2, deq, meta_ok, code_ok);
  if (!aok) {
    for (int j = 0; j < D / group; ++j) meta_ok[j] = 0;
    for (int i = 0; i < D; ++i) code_ok[i] = 0;
  }
}

void rqo_quantize_box_rows(const float* lo, const float* hi, const float* mid, int64_t n,
                           int D, int bits, int group, uint32_t* words, uint32_t* meta,
                           float* deq, uint8_t* meta_ok, uint8_t* code_ok) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r)
    rqo_quantize_box(lo + r * D, hi + r * D, mid + r * D, D, bits, group, words + r * W,
                     meta + r * G, deq + r * D, meta_ok + r * G, code_ok + r * D);
}

void rqo_encode_residual_box_rows(const float* lo, const float* hi, const float* mid,
                                  const float* ref, const float* mu, int64_t n, int D,
                                  int bits, int group, int unit_alpha, uint32_t* words,
                                  uint32_t* meta, uint16_t* alpha, float* zhat,
                                  uint8_t* alpha_ok, uint8_t* meta_ok, uint8_t* code_ok) {
  const int W = D * bits / 32, G = D / group;
  for (int64_t r = 0; r < n; ++r)
    rqo_encode_residual_box(lo + r * D, hi + r * D, mid + r * D, ref + r * D,
                            mu ? mu + r * D : NULL, D, bits, group, unit_alpha, words + r * W,
                            meta + r * G, alpha + r, zhat + r * D, alpha_ok + r,
                            meta_ok + r * G, code_ok + r * D);
}

/* ------------------------------------------------------------------------ */
/* Storage and access accounting [RQ §5.1, App. A.3, App. D]                */
/* ------------------------------------------------------------------------ */

double rqo_effective_bits(int L, const int* bits, const int* group, int D,
                          int meta_bits, int residual) {
  double total = 0.0;
  for (int r = 0; r < L; ++r)
    total += (double)bits[r] + (double)meta_bits / (double)group[r];
  if (residual) total += (double)(L - 1) * 16.0 / (double)D;
  return total / (double)L;
}

int64_t rqo_component_reads(int L, int chained) {
  /* One decode step over loops 0..L-1 [RQ §3.2, App. D].  The anchor loop
   * reads one component.  Under a shared anchor (First-loop, Last-loop)
   * every other loop reads the anchor and its own residual; under a chain
   * (Previous-loop, Next-loop) loop r reads its residual, every residual
   * between it and the anchor, and the anchor: 1 + its distance from the
   * anchor.  The count does not depend on which end holds the anchor, so
   * it is written for the anchor at L-1. */
  int64_t total = 0;
  for (int r = 0; r < L; ++r) {
    if (r == L - 1)
      total += 1;
    else if (!chained)
      total += 2;
    else
      total += (L - 1 - r) + 1;
  }
  return total;
}
