// rq_decode_common.cuh -- pieces shared by the decode kernels: the
// end-of-split reduction, the last-CTA merge with the current token and the
// final inverse rotation [RQ §4.1, §4.2 Decode, App. G.2].
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
#pragma once

#include <math.h>

#include "rq_internal.cuh"

namespace rq {

constexpr float kNegInf = -INFINITY;

// Exact small-integer -> float conversion: 0x4B000000 | c is 2^23 + c.
__device__ __forceinline__ float code_to_float(uint32_t c) {
  return __uint_as_float(0x4B000000u | c) - 8388608.0f;
}

__device__ __forceinline__ void unpack_meta(uint32_t mw, float& s, float& z) {
  const __half2 h = *reinterpret_cast<const __half2*>(&mw);
  const float2 f = __half22float2(h);
  s = f.x;
  z = f.y;
}

__device__ __forceinline__ int log2_pow2(int v) { return 31 - __clz(v); }

// In-place Hadamard butterflies (unnormalised) over D values in shared
// memory; every thread of the CTA must call it.
template <int D>
__device__ __forceinline__ void smem_fwht(float* v) {
  const int t = threadIdx.x;
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    if (t < D && (t & h) == 0) {
      const float a = v[t], b = v[t + h];
      v[t] = a + b;
      v[t + h] = a - b;
    }
    __syncthreads();
  }
}

// Rotated query in svec (which holds the bf16 query on entry), every thread
// of the CTA calls it.  Hadamard: the unnormalised butterflies, and the
// returned factor rot_scale normalises them.  Dense rotation [RQ App. G.2]
// (urot: this head's binary16 D x D matrix, row i = output channel i):
// U q~ with q~ the query rounded to binary16 and fp32 sums; returns 1.
template <int D>
__device__ __forceinline__ float rotate_query(float* svec, const uint16_t* urot,
                                              float rot_scale) {
  const int t = threadIdx.x;
  if (urot == nullptr) {
    smem_fwht<D>(svec);
    return rot_scale;
  }
  if (t < D) svec[t] = __half2float(__float2half_rn(svec[t]));
  __syncthreads();
  float a = 0.0f;
  if (t < D) {
    const uint4* row = reinterpret_cast<const uint4*>(urot + static_cast<size_t>(t) * D);
#pragma unroll 4
    for (int j8 = 0; j8 < D / 8; ++j8) {
      const uint4 w = __ldg(row + j8);
      const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 u = __half22float2(*reinterpret_cast<const __half2*>(&h[e]));
        a = fmaf(u.x, svec[8 * j8 + 2 * e], a);
        a = fmaf(u.y, svec[8 * j8 + 2 * e + 1], a);
      }
    }
  }
  __syncthreads();
  if (t < D) svec[t] = a;
  __syncthreads();
  return 1.0f;
}

// Sequence length of batch row b, clamped to [0, max_seq_len] and flagged.
__device__ __forceinline__ int seq_len_of(const int32_t* seq_lens, int b, int max_seq_len,
                                          uint32_t* err) {
  int n = seq_lens[b];
  if (n < 0 || n > max_seq_len) {
    if (threadIdx.x == 0) atomicOr(err, kErrSeqLen);
    n = n < 0 ? 0 : max_seq_len;
  }
  return n;
}

// End of a split.  Every thread of the CTA (NT threads) calls this.  Threads
// with slot >= 0 own the online-softmax state (m, l, acc[32]) of token slot
// `slot` for channels [32*slice, 32*slice+32).  The slots are reduced into one
// partial (m, l, acc[D]) in the workspace; the last CTA of the (batch, head)
// then merges every split with the current token and writes the output,
// applying H^T once when ROT.  `scratch` holds max(NSLOT*red_pitch<D>() +
// 2*NSLOT, 3*splits) floats.  `bad` (the same for every thread of the CTA)
// marks a split whose result is not valid (a bounded wait ran out, or a value
// left the accumulator range): it is counted in the upper half of the
// (batch, head)'s split counter, and the merging CTA then writes NaN to that
// (batch, head)'s output row instead of a partial sum.
//
// The slot reduction buffer keeps each slice's 32 channels in a block of 36
// floats (a slot is D/32 blocks): the 16-byte stores of the lanes of one
// quarter-warp (consecutive slices and slots) then fall in distinct bank
// groups.
constexpr int kRedSliceFloats = 36;
template <int D>
__host__ __device__ constexpr int red_pitch() { return (D / 32) * kRedSliceFloats; }

template <int D, int NT, int NSLOT, bool ROT>
__device__ __forceinline__ void finish_split(float m, float l, const float (&acc)[32], int slice,
                                             int slot, float* scratch, int bhi, int split,
                                             int splits, float* partials, uint32_t* counters,
                                             const uint16_t* q, const uint16_t* kcur,
                                             const uint16_t* vcur, float scale_log2,
                                             float rot_scale, float* out, float* svec,
                                             float* sred, bool bad,
                                             const uint16_t* urot = nullptr) {
  constexpr int RP = red_pitch<D>();
  float* red = scratch;                 // [NSLOT][D/32][36]
  float* mred = red + NSLOT * RP;       // [NSLOT]
  float* lred = mred + NSLOT;           // [NSLOT]
  const int t = threadIdx.x;
  if (slot >= 0 && slice == 0) {
    mred[slot] = m;
    lred[slot] = l;
  }
  __syncthreads();
  float M = kNegInf;
  for (int s = 0; s < NSLOT; ++s) M = fmaxf(M, mred[s]);
  if (slot >= 0) {
    const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - M);
    float4* dst = reinterpret_cast<float4*>(red + slot * RP + slice * kRedSliceFloats);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(acc[4 * i] * f, acc[4 * i + 1] * f, acc[4 * i + 2] * f,
                           acc[4 * i + 3] * f);
  }
  __syncthreads();
  float* part = partials + (static_cast<size_t>(bhi) * splits + split) * (D + 2);
  if (t < D) {
    float sum = 0.0f;
    const float* col = red + (t >> 5) * kRedSliceFloats + (t & 31);
    for (int s = 0; s < NSLOT; ++s) sum += col[s * RP];
    part[2 + t] = sum;
  }
  if (t == 0) {
    float L = 0.0f;
    for (int s = 0; s < NSLOT; ++s)
      L += (mred[s] == kNegInf) ? 0.0f : lred[s] * fast_exp2(mred[s] - M);
    part[0] = M;
    part[1] = L;
  }
  // Publish the partial, then count this split in (no waiting on other CTAs):
  // the CTA barrier orders every thread's partial writes before thread 0's
  // acquire-release add, which makes them visible with it (and, for the last
  // CTA, makes every other split's partial visible to it).
  __syncthreads();
  __shared__ uint32_t s_last, s_bad;
  if (t == 0) {
    // low 16 bits: splits counted in (splits <= 1024); high 16: bad splits
    const uint32_t inc = bad ? 0x10001u : 1u;
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(counters + bhi), "r"(inc) : "memory");
    s_last = ((old + inc) & 0xFFFFu) == static_cast<uint32_t>(splits);
    s_bad = (old + inc) >> 16;
  }
  __syncthreads();
  if (!s_last) return;
  if (s_bad != 0u) {   // a split of this (batch, head) is not valid
    if (t < D) out[static_cast<size_t>(bhi) * D + t] = __int_as_float(0x7FC00000);
    if (t == 0) counters[bhi] = 0u;
    return;
  }

  // ---- last CTA of this (batch, head): merge ----
  // Current token score q.k_cur, original domain [RQ §3.2, §4.2].
  float qk = 0.0f;
  if (t < D)
    qk = bf16_bits_to_f32(q[static_cast<size_t>(bhi) * D + t]) *
         bf16_bits_to_f32(kcur[static_cast<size_t>(bhi) * D + t]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
  if ((t & 31) == 0) sred[t >> 5] = qk;
  // Split headers (m, l) into shared memory (the scratch is free now).
  const float* pbase = partials + static_cast<size_t>(bhi) * splits * (D + 2);
  float* sm_m = scratch;              // [splits]
  float* sm_l = scratch + splits;     // [splits]
  float* sm_f = scratch + 2 * splits; // [splits]
  for (int s = t; s < splits; s += NT) {
    sm_m[s] = __ldcg(pbase + static_cast<size_t>(s) * (D + 2));
    sm_l[s] = __ldcg(pbase + static_cast<size_t>(s) * (D + 2) + 1);
  }
  __syncthreads();
  float s_cur = 0.0f;
  for (int w = 0; w < (D + 31) / 32; ++w) s_cur += sred[w];
  s_cur *= scale_log2;
  float Mx = s_cur;
  for (int s = 0; s < splits; ++s) Mx = fmaxf(Mx, sm_m[s]);
  for (int s = t; s < splits; s += NT)
    sm_f[s] = (sm_m[s] == kNegInf) ? 0.0f : fast_exp2(sm_m[s] - Mx);
  __syncthreads();
  float Lx = fast_exp2(s_cur - Mx);
  for (int s = 0; s < splits; ++s) Lx = fmaf(sm_l[s], sm_f[s], Lx);
  float ax = 0.0f;
  if (t < D) {
    const float* col = pbase + 2 + t;
    int s = 0;
    for (; s + 8 <= splits; s += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(col + static_cast<size_t>(s + u) * (D + 2));
#pragma unroll
      for (int u = 0; u < 8; ++u) ax = fmaf(v[u], sm_f[s + u], ax);
    }
    for (; s < splits; ++s) ax = fmaf(__ldcg(col + static_cast<size_t>(s) * (D + 2)), sm_f[s], ax);
  }
  __syncthreads();   // everyone is done reading svec / the scratch
  if (t < D) svec[t] = ax;
  __syncthreads();
  // Back to the original domain: the Hadamard butterflies, or U_V^T of the
  // fp32 value sum under a dense rotation [RQ App. G.2] (column t of U).
  float dv = 0.0f;
  if (urot != nullptr) {
    if (t < D)
      for (int j = 0; j < D; ++j)
        dv = fmaf(__half2float(__ushort_as_half(__ldg(urot + static_cast<size_t>(j) * D + t))),
                  svec[j], dv);
  } else if constexpr (ROT) {
    smem_fwht<D>(svec);
  }
  if (t < D) {
    const float pc = fast_exp2(s_cur - Mx);
    const float v = urot != nullptr ? dv : (ROT ? svec[t] * rot_scale : svec[t]);
    out[static_cast<size_t>(bhi) * D + t] =
        (v + pc * bf16_bits_to_f32(vcur[static_cast<size_t>(bhi) * D + t])) / Lx;
  }
  if (t == 0) counters[bhi] = 0u;   // ready for the next call
}

}  // namespace rq
