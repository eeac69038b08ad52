// rq_decode.cu -- split-K decode attention over the packed ResidualQuant
// cache, and the uncompressed BF16 decode kernel on the same engine.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// Work decomposition: one CTA (128 threads) per (batch*head, split); a split
// is a contiguous range of past tokens.  Each CTA streams its range in chunks
// of kChunk tokens: thread 0 issues one bulk asynchronous copy per packed
// array (codes, metadata, LS coefficients of every component, K and V) into
// an S-stage shared-memory ring, completing on a per-stage mbarrier; all
// threads consume a stage, synchronise, and thread 0 refills it.
//
// Compute [RQ §4.1, App. G.2]: q' = H q is formed once per CTA and the
// score of a past token is q'.Z^_K = sum_c kappa_c (s~ q'.code + z~ sum q'),
// kappa = product of the LS coefficients along the reference chain
// (kappa = 1 for the loop's own residual, alpha~ for the shared anchor).
// Values are accumulated in the rotated domain with an online softmax in
// fp32 (exp2 with log2(e) folded into q').  A token is owned by P = D/32
// lanes, each holding 32 channels.  Partials (m, l, acc[D]) of a split go to
// the workspace; the last CTA of a (batch, head) -- elected by an atomic
// counter, no waiting -- merges the splits and the current token's bf16
// k/v [RQ §4.2 Decode], applies H^T once and writes the output.
#include <math.h>

#include "rq_internal.cuh"

namespace rq {
namespace {

constexpr float kNegInf = -INFINITY;

template <int D>
struct Geom {
  static constexpr int P = D / 32;            // lanes per token
  static constexpr int TPW = 32 / P;          // tokens per warp pass
  static constexpr int TPC = 4 * TPW;         // tokens per CTA pass
  static constexpr int TT = kChunk / TPC;     // tokens per thread per chunk
  static constexpr int NSLOT = kDecodeThreads / P;
};

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

// Per-component shared-memory offsets inside one pipeline stage.
struct StageMap {
  uint32_t codes[2][RQ_MAX_LOOPS];
  uint32_t meta[2][RQ_MAX_LOOPS];
  uint32_t alpha[2][RQ_MAX_LOOPS];
  uint32_t bytes;
};

__host__ __device__ inline void build_stage_map(const DecodeParams& p, int D,
                                                StageMap& m) {
  uint32_t off = 0;
  for (int side = 0; side < 2; ++side) {
    const Comp* cs = side == 0 ? p.k : p.v;
    for (int c = 0; c < p.ncomp; ++c) {
      m.codes[side][c] = off;
      off += kChunk * (D * cs[c].bits / 32) * 4;
      m.meta[side][c] = off;
      off += kChunk * (D / cs[c].group) * 4;
      m.alpha[side][c] = off;
      if (cs[c].alpha != nullptr) off += kChunk * 2;
    }
  }
  m.bytes = off;
}

// q'.D(c) over this lane's 32 channels of one token of one component:
// s~ * sum q'_i c_i + z~ * sum q'_i per group part.
template <int BITS>
__device__ __forceinline__ float comp_dot(const uint32_t* cw, const uint32_t* mrow,
                                          int slice, int gshift, const float (&q)[32],
                                          float qsa, float qsb) {
  constexpr int PER_WORD = 32 / BITS;
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  uint32_t w[BITS];
  if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(cw);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(cw);
    w[0] = v.x; w[1] = v.y;
  }
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) {
    const uint32_t c = (w[ch / PER_WORD] >> (BITS * (ch % PER_WORD))) & QMAX;
    if (ch < 16)
      a0 = fmaf(q[ch], code_to_float(c), a0);
    else
      a1 = fmaf(q[ch], code_to_float(c), a1);
  }
  float s0, z0, s1, z1;
  if (gshift >= 5) {
    unpack_meta(mrow[(slice * 32) >> gshift], s0, z0);
    return s0 * (a0 + a1) + z0 * (qsa + qsb);
  }
  const uint2 mw = *reinterpret_cast<const uint2*>(mrow + slice * 2);
  unpack_meta(mw.x, s0, z0);
  unpack_meta(mw.y, s1, z1);
  return s0 * a0 + z0 * qsa + (s1 * a1 + z1 * qsb);
}

// acc += pk * D(c) over this lane's 32 channels; the offsets go to cst0/cst1.
template <int BITS>
__device__ __forceinline__ void comp_acc(const uint32_t* cw, const uint32_t* mrow,
                                         int slice, int gshift, float pk, float (&acc)[32],
                                         float& cst0, float& cst1) {
  constexpr int PER_WORD = 32 / BITS;
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  uint32_t w[BITS];
  if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(cw);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(cw);
    w[0] = v.x; w[1] = v.y;
  }
  float s0, z0, s1, z1;
  if (gshift >= 5) {
    unpack_meta(mrow[(slice * 32) >> gshift], s0, z0);
    s1 = s0;
    z1 = z0;
  } else {
    const uint2 mw = *reinterpret_cast<const uint2*>(mrow + slice * 2);
    unpack_meta(mw.x, s0, z0);
    unpack_meta(mw.y, s1, z1);
  }
  const float w0 = pk * s0, w1 = pk * s1;
  cst0 = fmaf(pk, z0, cst0);
  cst1 = fmaf(pk, z1, cst1);
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) {
    const uint32_t c = (w[ch / PER_WORD] >> (BITS * (ch % PER_WORD))) & QMAX;
    acc[ch] = fmaf(ch < 16 ? w0 : w1, code_to_float(c), acc[ch]);
  }
}

__device__ __forceinline__ int log2_pow2(int v) { return 31 - __clz(v); }

// In-place normalised-free Hadamard butterflies over D values in shared
// memory, D threads participating (thread t < D).
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

// Reduction of the per-slot online-softmax states of a CTA into one partial
// (m, l, acc[D]) in the workspace, then the last-CTA merge of all splits with
// the current token.  `stage_mem` is free scratch of at least
// (NSLOT*D + 2*NSLOT) floats.  ROT: apply H^T to the merged accumulator.
template <int D, bool ROT>
__device__ __forceinline__ void finish(float m, float l, float (&acc)[32], int slice,
                                       int slot, float* stage_mem, int bhi, int split,
                                       int splits, float* partials, uint32_t* counters,
                                       const uint16_t* q, const uint16_t* kcur,
                                       const uint16_t* vcur, float scale_log2,
                                       float rot_scale, float* out, float* svec,
                                       float* sred) {
  using G = Geom<D>;
  float* red = stage_mem;                       // [NSLOT][D]
  float* mred = red + G::NSLOT * D;             // [NSLOT]
  float* lred = mred + G::NSLOT;                // [NSLOT]
  const int t = threadIdx.x;
  if (slice == 0) {
    mred[slot] = m;
    lred[slot] = l;
  }
  __syncthreads();
  float M = kNegInf;
  for (int s = 0; s < G::NSLOT; ++s) M = fmaxf(M, mred[s]);
  const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - M);
  float4* dst = reinterpret_cast<float4*>(red + slot * D + slice * 32);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    dst[i] = make_float4(acc[4 * i] * f, acc[4 * i + 1] * f, acc[4 * i + 2] * f,
                         acc[4 * i + 3] * f);
  __syncthreads();
  float* part = partials + (static_cast<size_t>(bhi) * splits + split) * (D + 2);
  if (t < D) {
    float sum = 0.0f;
    for (int s = 0; s < G::NSLOT; ++s) sum += red[s * D + t];
    part[2 + t] = sum;
  }
  if (t == 0) {
    float L = 0.0f;
    for (int s = 0; s < G::NSLOT; ++s)
      L += (mred[s] == kNegInf) ? 0.0f : lred[s] * fast_exp2(mred[s] - M);
    part[0] = M;
    part[1] = L;
  }
  // Publish the partial, then count this split in.
  __threadfence();
  __syncthreads();
  __shared__ uint32_t s_last;
  if (t == 0) s_last = (atomicAdd(counters + bhi, 1u) == static_cast<uint32_t>(splits - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of this (batch, head): merge ----
  // Current token score q.k_cur in the original domain [RQ §3.2, §4.2].
  float qk = 0.0f;
  if (t < D) qk = bf16_bits_to_f32(q[static_cast<size_t>(bhi) * D + t]) *
                  bf16_bits_to_f32(kcur[static_cast<size_t>(bhi) * D + t]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
  if ((t & 31) == 0) sred[t >> 5] = qk;
  __syncthreads();
  const float s_cur = (sred[0] + sred[1] + sred[2] + sred[3]) * scale_log2;
  const float* pbase = partials + static_cast<size_t>(bhi) * splits * (D + 2);
  float Mx = s_cur;
  for (int s = 0; s < splits; ++s) Mx = fmaxf(Mx, __ldcg(pbase + s * (D + 2)));
  float Lx = fast_exp2(s_cur - Mx);
  float ax = 0.0f;
  for (int s = 0; s < splits; ++s) {
    const float ms = __ldcg(pbase + s * (D + 2));
    if (ms == kNegInf) continue;
    const float fs = fast_exp2(ms - Mx);
    Lx += __ldcg(pbase + s * (D + 2) + 1) * fs;
    if (t < D) ax += __ldcg(pbase + s * (D + 2) + 2 + t) * fs;
  }
  if (t < D) svec[t] = ax;
  __syncthreads();
  if constexpr (ROT) smem_fwht<D>(svec);
  if (t < D) {
    const float pc = fast_exp2(s_cur - Mx);
    const float v = ROT ? svec[t] * rot_scale : svec[t];
    out[static_cast<size_t>(bhi) * D + t] =
        (v + pc * bf16_bits_to_f32(vcur[static_cast<size_t>(bhi) * D + t])) / Lx;
  }
  if (t == 0) counters[bhi] = 0u;   // ready for the next call
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

template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  using G = Geom<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t full_bar[8];
  __shared__ StageMap map;
  __shared__ float svec[D];
  __shared__ float sred[4];
  __shared__ int s_abort;

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int slice = lane % G::P;
  const int tw = lane / G::P;
  const int slot = warp * G::TPW + tw;
  const int split = blockIdx.x;
  const int bhi = blockIdx.y;
  const int b = bhi / p.heads;
  const int S = p.stages;

  const int n = seq_len_of(p.seq_lens, b, p.max_seq_len, p.err);
  const int t_begin = split * p.chunks_per_split * kChunk;
  const int t_end = min(n, t_begin + p.chunks_per_split * kChunk);
  const int nchunks = t_end > t_begin ? (t_end - t_begin + kChunk - 1) / kChunk : 0;

  if (t == 0) {
    build_stage_map(p, D, map);
    for (int s = 0; s < S; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
    s_abort = 0;
  }
  // Rotated, pre-scaled query q' = H q * scale * log2(e).
  if (t < D) svec[t] = bf16_bits_to_f32(p.q[static_cast<size_t>(bhi) * D + t]);
  __syncthreads();

  const size_t row0 = static_cast<size_t>(bhi) * p.tstride;
  auto issue = [&](int i) {
    const int s = i % S;
    const int t0 = t_begin + i * kChunk;
    const int nt = min(kChunk, t_end - t0);
    const int ntc = (nt + 7) & ~7;   // 16-byte granules of the bf16 coefficients
    unsigned char* st = smem + static_cast<size_t>(s) * p.stage_bytes;
    uint32_t bytes = 0;
    for (int side = 0; side < 2; ++side) {
      const Comp* cs = side == 0 ? p.k : p.v;
      for (int c = 0; c < p.ncomp; ++c) {
        bytes += ntc * (D * cs[c].bits / 32) * 4 + ntc * (D / cs[c].group) * 4;
        if (cs[c].alpha != nullptr) bytes += ntc * 2;
      }
    }
    mbar_arrive_expect_tx(&full_bar[s], bytes);
    for (int side = 0; side < 2; ++side) {
      const Comp* cs = side == 0 ? p.k : p.v;
      for (int c = 0; c < p.ncomp; ++c) {
        const int wpr = D * cs[c].bits / 32, gpr = D / cs[c].group;
        bulk_copy_g2s(st + map.codes[side][c], cs[c].codes + (row0 + t0) * wpr,
                      ntc * wpr * 4, &full_bar[s]);
        bulk_copy_g2s(st + map.meta[side][c], cs[c].meta + (row0 + t0) * gpr,
                      ntc * gpr * 4, &full_bar[s]);
        if (cs[c].alpha != nullptr)
          bulk_copy_g2s(st + map.alpha[side][c], cs[c].alpha + row0 + t0, ntc * 2,
                        &full_bar[s]);
      }
    }
  };
  int issued = 0;
  if (t == 0) {
    for (; issued < min(S, nchunks); ++issued) issue(issued);
  }
  smem_fwht<D>(svec);
  float q[32];
  float qsa = 0.0f, qsb = 0.0f;
  {
    const float sc = p.rot_scale * p.scale_log2;
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) {
      q[ch] = svec[slice * 32 + ch] * sc;
      if (ch < 16) qsa += q[ch]; else qsb += q[ch];
    }
  }

  float m = kNegInf, l = 0.0f;
  float acc[32];
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) acc[ch] = 0.0f;
  float cst0 = 0.0f, cst1 = 0.0f;

  int i = 0;
  for (; i < nchunks; ++i) {
    const int s = i % S;
    if (!mbar_wait(&full_bar[s], (i / S) & 1, p.err)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    const unsigned char* st = smem + static_cast<size_t>(s) * p.stage_bytes;
    const int nt = min(kChunk, t_end - (t_begin + i * kChunk));

    // ---- scores ----
    float sc[G::TT];
#pragma unroll
    for (int tt = 0; tt < G::TT; ++tt) {
      const int j = tt * G::TPC + warp * G::TPW + tw;
      float part = 0.0f, kappa = 1.0f;
      for (int c = 0; c < p.ncomp; ++c) {
        const int bits = p.k[c].bits;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(st + map.codes[0][c]) +
                             j * (D * bits / 32) + slice * bits;
        const uint32_t* mr = reinterpret_cast<const uint32_t*>(st + map.meta[0][c]) +
                             j * (D / p.k[c].group);
        const float d = (bits == 4) ? comp_dot<4>(cw, mr, slice, log2_pow2(p.k[c].group), q, qsa, qsb)
                                    : comp_dot<2>(cw, mr, slice, log2_pow2(p.k[c].group), q, qsa, qsb);
        part = fmaf(kappa, d, part);
        if (c + 1 < p.ncomp)
          kappa *= bf16_bits_to_f32(
              reinterpret_cast<const uint16_t*>(st + map.alpha[0][c])[j]);
      }
#pragma unroll
      for (int off = G::P / 2; off >= 1; off >>= 1)
        part += __shfl_xor_sync(0xffffffffu, part, off);
      sc[tt] = (j < nt) ? part : kNegInf;
    }
    // ---- online softmax (per slot) ----
    float mc = sc[0];
#pragma unroll
    for (int tt = 1; tt < G::TT; ++tt) mc = fmaxf(mc, sc[tt]);
    if (mc > m) {
      const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - mc);
      l *= f;
      cst0 *= f;
      cst1 *= f;
#pragma unroll
      for (int ch = 0; ch < 32; ++ch) acc[ch] *= f;
      m = mc;
    }
    // ---- values ----
#pragma unroll
    for (int tt = 0; tt < G::TT; ++tt) {
      const int j = tt * G::TPC + warp * G::TPW + tw;
      if (sc[tt] == kNegInf) continue;
      const float pt = fast_exp2(sc[tt] - m);
      l += pt;
      float kappa = pt;
      for (int c = 0; c < p.ncomp; ++c) {
        const int bits = p.v[c].bits;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(st + map.codes[1][c]) +
                             j * (D * bits / 32) + slice * bits;
        const uint32_t* mr = reinterpret_cast<const uint32_t*>(st + map.meta[1][c]) +
                             j * (D / p.v[c].group);
        if (bits == 4)
          comp_acc<4>(cw, mr, slice, log2_pow2(p.v[c].group), kappa, acc, cst0, cst1);
        else
          comp_acc<2>(cw, mr, slice, log2_pow2(p.v[c].group), kappa, acc, cst0, cst1);
        if (c + 1 < p.ncomp)
          kappa *= bf16_bits_to_f32(
              reinterpret_cast<const uint16_t*>(st + map.alpha[1][c])[j]);
      }
    }
    __syncthreads();   // stage s fully consumed
    if (t == 0 && issued < nchunks) issue(issued++);
  }

  if (s_abort) {
    // Wait (bounded) for copies still in flight before the stages are reused
    // as scratch or the CTA exits; contribute nothing.
    if (t == 0) {
      // chunks before i were consumed; i .. issued-1 may still be in flight
      for (int k = i; k < issued; ++k) (void)mbar_wait(&full_bar[k % S], (k / S) & 1, p.err);
    }
    __syncthreads();
    m = kNegInf;
    l = 0.0f;
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) acc[ch] = 0.0f;
    cst0 = cst1 = 0.0f;
  }
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) acc[ch] += (ch < 16) ? cst0 : cst1;
  __syncthreads();
  finish<D, true>(m, l, acc, slice, slot, reinterpret_cast<float*>(smem), bhi, split,
                  p.splits, p.partials, p.counters, p.q, p.kcur, p.vcur, p.scale_log2,
                  p.rot_scale, p.out, svec, sred);
}

// Uncompressed bf16 rows: K and V [B*H][tstride][D].
template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_bf16_kernel(const __grid_constant__ DecodeBf16Params p) {
  using G = Geom<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t full_bar[8];
  __shared__ float svec[D];
  __shared__ float sred[4];
  __shared__ int s_abort;

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int slice = lane % G::P;
  const int tw = lane / G::P;
  const int slot = warp * G::TPW + tw;
  const int split = blockIdx.x;
  const int bhi = blockIdx.y;
  const int b = bhi / p.heads;
  const int S = p.stages;
  constexpr uint32_t kRowBytes = D * 2;

  const int n = seq_len_of(p.seq_lens, b, p.max_seq_len, p.err);
  const int t_begin = split * p.chunks_per_split * kChunk;
  const int t_end = min(n, t_begin + p.chunks_per_split * kChunk);
  const int nchunks = t_end > t_begin ? (t_end - t_begin + kChunk - 1) / kChunk : 0;

  if (t == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
    s_abort = 0;
  }
  __syncthreads();
  const size_t row0 = static_cast<size_t>(bhi) * p.tstride;
  auto issue = [&](int i) {
    const int s = i % S;
    const int t0 = t_begin + i * kChunk;
    const int nt = min(kChunk, t_end - t0);
    unsigned char* st = smem + static_cast<size_t>(s) * p.stage_bytes;
    mbar_arrive_expect_tx(&full_bar[s], 2u * nt * kRowBytes);
    bulk_copy_g2s(st, p.k + (row0 + t0) * D, nt * kRowBytes, &full_bar[s]);
    bulk_copy_g2s(st + kChunk * kRowBytes, p.v + (row0 + t0) * D, nt * kRowBytes,
                  &full_bar[s]);
  };
  int issued = 0;
  if (t == 0) {
    for (; issued < min(S, nchunks); ++issued) issue(issued);
  }
  float q[32];
  {
    const uint16_t* qr = p.q + static_cast<size_t>(bhi) * D + slice * 32;
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) q[ch] = bf16_bits_to_f32(qr[ch]) * p.scale_log2;
  }
  float m = kNegInf, l = 0.0f;
  float acc[32];
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) acc[ch] = 0.0f;

  int i = 0;
  for (; i < nchunks; ++i) {
    const int s = i % S;
    if (!mbar_wait(&full_bar[s], (i / S) & 1, p.err)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    const unsigned char* st = smem + static_cast<size_t>(s) * p.stage_bytes;
    const int nt = min(kChunk, t_end - (t_begin + i * kChunk));
    float sc[G::TT];
#pragma unroll
    for (int tt = 0; tt < G::TT; ++tt) {
      const int j = tt * G::TPC + warp * G::TPW + tw;
      const uint4* kr = reinterpret_cast<const uint4*>(st + j * kRowBytes + slice * 64);
      float part = 0.0f;
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const uint4 v = kr[i4];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          part = fmaf(q[i4 * 8 + 2 * e], __uint_as_float(w[e] << 16), part);
          part = fmaf(q[i4 * 8 + 2 * e + 1], __uint_as_float(w[e] & 0xFFFF0000u), part);
        }
      }
#pragma unroll
      for (int off = G::P / 2; off >= 1; off >>= 1)
        part += __shfl_xor_sync(0xffffffffu, part, off);
      sc[tt] = (j < nt) ? part : kNegInf;
    }
    float mc = sc[0];
#pragma unroll
    for (int tt = 1; tt < G::TT; ++tt) mc = fmaxf(mc, sc[tt]);
    if (mc > m) {
      const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - mc);
      l *= f;
#pragma unroll
      for (int ch = 0; ch < 32; ++ch) acc[ch] *= f;
      m = mc;
    }
#pragma unroll
    for (int tt = 0; tt < G::TT; ++tt) {
      const int j = tt * G::TPC + warp * G::TPW + tw;
      if (sc[tt] == kNegInf) continue;
      const float pt = fast_exp2(sc[tt] - m);
      l += pt;
      const uint4* vr =
          reinterpret_cast<const uint4*>(st + kChunk * kRowBytes + j * kRowBytes + slice * 64);
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const uint4 v = vr[i4];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[i4 * 8 + 2 * e] = fmaf(pt, __uint_as_float(w[e] << 16), acc[i4 * 8 + 2 * e]);
          acc[i4 * 8 + 2 * e + 1] =
              fmaf(pt, __uint_as_float(w[e] & 0xFFFF0000u), acc[i4 * 8 + 2 * e + 1]);
        }
      }
    }
    __syncthreads();
    if (t == 0 && issued < nchunks) issue(issued++);
  }
  if (s_abort) {
    if (t == 0) {
      for (int k = i; k < issued; ++k) (void)mbar_wait(&full_bar[k % S], (k / S) & 1, p.err);
    }
    __syncthreads();
    m = kNegInf;
    l = 0.0f;
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) acc[ch] = 0.0f;
  }
  __syncthreads();
  finish<D, false>(m, l, acc, slice, slot, reinterpret_cast<float*>(smem), bhi, split,
                   p.splits, p.partials, p.counters, p.q, p.kcur, p.vcur, p.scale_log2,
                   1.0f, p.out, svec, sred);
}

template <int D>
size_t scratch_bytes() {
  return (Geom<D>::NSLOT * D + 2 * Geom<D>::NSLOT) * sizeof(float);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

uint32_t decode_stage_bytes(const DecodeParams& p, int D) {
  StageMap m;
  build_stage_map(p, D, m);
  return m.bytes;
}

size_t decode_dyn_smem(int D, int stages, uint32_t stage_bytes) {
  const size_t ring = static_cast<size_t>(stages) * stage_bytes;
  const size_t scr = D == 64 ? scratch_bytes<64>() : scratch_bytes<128>();
  return ring > scr ? ring : scr;
}

cudaError_t decode_occupancy(int D, bool bf16, size_t dyn_smem, int* ctas_per_sm) {
  cudaError_t e;
  if (bf16) {
    if (D == 64) {
      e = set_smem(decode_bf16_kernel<64>, dyn_smem);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_bf16_kernel<64>,
                                                          kDecodeThreads, dyn_smem);
    } else {
      e = set_smem(decode_bf16_kernel<128>, dyn_smem);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_bf16_kernel<128>,
                                                          kDecodeThreads, dyn_smem);
    }
  } else {
    if (D == 64) {
      e = set_smem(decode_kernel<64>, dyn_smem);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_kernel<64>,
                                                          kDecodeThreads, dyn_smem);
    } else {
      e = set_smem(decode_kernel<128>, dyn_smem);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_kernel<128>,
                                                          kDecodeThreads, dyn_smem);
    }
  }
  return e;
}

cudaError_t launch_decode(const DecodeParams& p, int D, cudaStream_t s) {
  const size_t dyn = decode_dyn_smem(D, p.stages, p.stage_bytes);
  const dim3 grid(p.splits, p.bh);
  if (D == 64) {
    cudaError_t e = set_smem(decode_kernel<64>, dyn);
    if (e != cudaSuccess) return e;
    decode_kernel<64><<<grid, kDecodeThreads, dyn, s>>>(p);
  } else if (D == 128) {
    cudaError_t e = set_smem(decode_kernel<128>, dyn);
    if (e != cudaSuccess) return e;
    decode_kernel<128><<<grid, kDecodeThreads, dyn, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_bf16(const DecodeBf16Params& p, int D, cudaStream_t s) {
  const size_t dyn = decode_dyn_smem(D, p.stages, p.stage_bytes);
  const dim3 grid(p.splits, p.bh);
  if (D == 64) {
    cudaError_t e = set_smem(decode_bf16_kernel<64>, dyn);
    if (e != cudaSuccess) return e;
    decode_bf16_kernel<64><<<grid, kDecodeThreads, dyn, s>>>(p);
  } else if (D == 128) {
    cudaError_t e = set_smem(decode_bf16_kernel<128>, dyn);
    if (e != cudaSuccess) return e;
    decode_bf16_kernel<128><<<grid, kDecodeThreads, dyn, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rq
