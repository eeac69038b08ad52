// rq_decode_fast.cu -- warp-specialised split-K decode attention for the
// packed ResidualQuant cache (compile-time component layouts) and for the
// uncompressed BF16 baseline.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// CTA = 8 compute warps + 1 producer warp.  The producer streams a split's
// token range in chunks with bulk asynchronous copies (one per packed array)
// into an S-stage shared-memory ring: full[s] completes on the copies' byte
// count, empty[s] when all compute warps are done with the stage.
//
// Scores [RQ §4.1, App. G.2]: q' = H q (pre-scaled by softmax scale and
// log2 e) is held as 16-bit fixed point, q' ~= sigma * (256 h + l) with
// int8 limbs h, l, so q'.codes over a group is two integer dot products
// (dp4a) of the unpacked code bytes with the limbs; the score of a token is
// sigma * sum_c kappa_c (s~_c * dot_c + z~_c * sum q~), kappa the product of
// the LS coefficients along the reference chain.
// Values: codes are turned into exact floats c * 2^p by OR-ing them into the
// mantissa of 2^23 and subtracting 2^23 (packed fp32 pairs), and accumulated
// with packed fp32 FMAs against weights p_t * kappa * s~ * 2^-p; the offsets
// z~ go to one accumulator per 16 channels.  Accumulation is in the rotated
// domain; H^T is applied once in the merge.
#include "rq_decode_common.cuh"

namespace rq {
namespace {

constexpr int kWarps = 8;                      // BF16 kernel: compute warps per CTA
constexpr int kThreads = (kWarps + 1) * 32;    // + producer warp
constexpr int kMaxRing = 4;

constexpr int kCWarps = 4;                     // compressed kernel: warps per CTA
constexpr int kCThreads = kCWarps * 32;
constexpr int kCChunk = 64;                    // tokens per stage
constexpr int kCMinCtas = 5;                   // register target: CTAs per SM
constexpr size_t kCRingBudget = 40 * 1024;     // stage ring per CTA (several CTAs per SM)
constexpr size_t kMergeScratch = 3 * 1024 * sizeof(float);   // split headers, up to 1024 splits

template <int D_, int NC_, int RB_, int RG_, int AB_, int AG_>
struct Spec {
  static constexpr int D = D_, NC = NC_, TC = kCChunk;
  __host__ __device__ static constexpr int bits(int c) { return c == NC_ - 1 ? AB_ : RB_; }
  __host__ __device__ static constexpr int group(int c) { return c == NC_ - 1 ? AG_ : RG_; }
  __host__ __device__ static constexpr bool has_alpha(int c) { return c != NC_ - 1; }
  __host__ __device__ static constexpr int wpr(int c) { return D_ * bits(c) / 32; }
  __host__ __device__ static constexpr int gpr(int c) { return D_ / group(c); }
  __host__ __device__ static constexpr uint32_t comp_bytes(int c) {
    return TC * (wpr(c) * 4 + gpr(c) * 4 + (has_alpha(c) ? 2 : 0));
  }
  __host__ __device__ static constexpr uint32_t side_bytes() {
    uint32_t s = 0;
    for (int c = 0; c < NC_; ++c) s += comp_bytes(c);
    return s;
  }
  __host__ __device__ static constexpr uint32_t stage_bytes() { return 2 * side_bytes(); }
  __host__ __device__ static constexpr uint32_t codes_off(int side, int c) {
    uint32_t o = side * side_bytes();
    for (int k = 0; k < c; ++k) o += comp_bytes(k);
    return o;
  }
  __host__ __device__ static constexpr uint32_t meta_off(int side, int c) {
    return codes_off(side, c) + TC * wpr(c) * 4;
  }
  __host__ __device__ static constexpr uint32_t alpha_off(int side, int c) {
    return meta_off(side, c) + TC * gpr(c) * 4;
  }
};

// Fixed-point rotated query of one lane's 32 channels as int8 limb bytes in
// the quad order of the unpacked codes: quad (k, s) holds channels
// 16k + s + {0, 4, 8, 12} (the same for 2-bit and 4-bit codes).
struct QLimbs {
  int h[2][4], l[2][4];
  float sq[2];   // sum of q~ over channels 0-15 / 16-31
};

// Unnormalised Hadamard butterflies over a row held by P = D/32 lanes, lane
// `slice` holding channels 32*slice .. 32*slice+31 (stages h = 1..16 inside
// the lane, then across lanes by xor-shuffles).
template <int D>
__device__ __forceinline__ void fwht_lanes(float (&z)[32], int slice) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = z[j], b = z[j + h];
        z[j] = a + b;
        z[j + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int hl = 1; hl < D / 32; hl <<= 1) {
    const bool upper = (slice & hl) != 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, z[k], hl);
      z[k] = upper ? o - z[k] : z[k] + o;
    }
  }
}

__device__ __forceinline__ int pack_bytes(int a, int b, int c, int d) {
  return (a & 0xFF) | ((b & 0xFF) << 8) | ((c & 0xFF) << 16) | (d << 24);
}

__device__ __forceinline__ void build_limbs(const float* qrow, float inv_sigma, QLimbs& ql) {
  int hi[32], lo[32];
  float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int qt = __float2int_rn(qrow[i] * inv_sigma);   // |qt| <= 32639
    const int h = (qt + 128) >> 8;
    hi[i] = h;
    lo[i] = qt - 256 * h;
    if (i < 16) s0 += static_cast<float>(qt); else s1 += static_cast<float>(qt);
  }
  ql.sq[0] = s0;
  ql.sq[1] = s1;
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int b = 16 * k + s;
      ql.h[k][s] = pack_bytes(hi[b], hi[b + 4], hi[b + 8], hi[b + 12]);
      ql.l[k][s] = pack_bytes(lo[b], lo[b + 4], lo[b + 8], lo[b + 12]);
    }
}

// q~ . D(c) over one lane's 32 channels of token j of a component, in sigma
// units: sum over group parts of s~ * (q~ . codes) + z~ * (sum q~).
template <int D, int BITS, int G>
__device__ __forceinline__ float kdot(const unsigned char* codes, const unsigned char* meta, int j,
                                      int slice, const QLimbs& ql) {
  constexpr int WPR = D * BITS / 32, GPR = D / G;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes) + j * WPR + slice * BITS;
  int ah[2] = {0, 0}, al[2] = {0, 0};   // per 16-channel block
  if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(cw);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int k = k4 >> 1, h = k4 & 1;
      const int lo = static_cast<int>(w[k4] & 0x0F0F0F0Fu);          // quad s = 2h
      const int hi = static_cast<int>((w[k4] >> 4) & 0x0F0F0F0Fu);   // quad s = 2h + 1
      ah[k] = __dp4a(ql.h[k][2 * h], lo, ah[k]);
      al[k] = __dp4a(ql.l[k][2 * h], lo, al[k]);
      ah[k] = __dp4a(ql.h[k][2 * h + 1], hi, ah[k]);
      al[k] = __dp4a(ql.l[k][2 * h + 1], hi, al[k]);
    }
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(cw);
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int x = static_cast<int>((w[k] >> (2 * s)) & 0x03030303u);
        ah[k] = __dp4a(ql.h[k][s], x, ah[k]);
        al[k] = __dp4a(ql.l[k][s], x, al[k]);
      }
  }
  const uint32_t* mr = reinterpret_cast<const uint32_t*>(meta) + j * GPR;
  float s0, z0;
  if constexpr (G >= 32) {
    unpack_meta(mr[(slice * 32) / G], s0, z0);
    return s0 * static_cast<float>((ah[0] + ah[1]) * 256 + (al[0] + al[1])) +
           z0 * (ql.sq[0] + ql.sq[1]);
  } else {
    float s1, z1;
    const uint2 mw = *reinterpret_cast<const uint2*>(mr + slice * 2);
    unpack_meta(mw.x, s0, z0);
    unpack_meta(mw.y, s1, z1);
    return s0 * static_cast<float>(ah[0] * 256 + al[0]) + z0 * ql.sq[0] +
           (s1 * static_cast<float>(ah[1] * 256 + al[1]) + z1 * ql.sq[1]);
  }
}

// Value path.  A code masked out of its word with the rest of the register
// (and so the exponent field) zero is the exact fp32 subnormal c * 2^(p-149),
// p its bit position (p + bits <= 23).  One FFMA with the fp32 weight
// w_p = p_t * kappa * s~ * 2^(kPosBias - p) adds p_t * kappa * s~ * c * 2^-40
// to the channel's accumulator: one mask and one FMA per code, fp32 weights.
constexpr int kPosBias = 109;                        // 2^(109 - p) <= 2^109 stays finite
constexpr float kValueUnscale = 1099511627776.0f;    // 2^(149 - kPosBias) = 2^40
constexpr float kWeightMax = 262144.0f;              // 2^18: weights above this are flagged

__device__ __forceinline__ float pow2_bias(int pos) {
  return __uint_as_float(static_cast<uint32_t>(127 + kPosBias - pos) << 23);
}

// acc += w * D(c) over one lane's 32 channels of token j (codes part; the z~
// offsets go to cst per 16-channel half).  pk = p_t * kappa.
template <int D, int BITS, int G>
__device__ __forceinline__ void vacc(const unsigned char* codes, const unsigned char* meta, int j,
                                     int slice, float pk, float (&acc)[32], float (&cst)[2],
                                     uint32_t& range_err) {
  constexpr int WPR = D * BITS / 32, GPR = D / G;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes) + j * WPR + slice * BITS;
  const uint32_t* mr = reinterpret_cast<const uint32_t*>(meta) + j * GPR;
  float sc[2], zc[2];
  if constexpr (G >= 32) {
    unpack_meta(mr[(slice * 32) / G], sc[0], zc[0]);
    sc[1] = sc[0];
    zc[1] = zc[0];
  } else {
    const uint2 mw = *reinterpret_cast<const uint2*>(mr + slice * 2);
    unpack_meta(mw.x, sc[0], zc[0]);
    unpack_meta(mw.y, sc[1], zc[1]);
  }
  constexpr int NPOS = BITS == 2 ? 8 : 4;   // positions 0,2,..,14 or 0,4,8,12 (after >>16)
  constexpr int NW = G >= 32 ? 1 : 2;       // distinct weights per lane
  float ws[2][NPOS];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    cst[h] = fmaf(pk, zc[h], cst[h]);
    if (h >= NW) continue;
    float w = pk * sc[h];
    if (!(fabsf(w) <= kWeightMax)) {
      range_err = 1u;
      w = 0.0f;
    }
#pragma unroll
    for (int q = 0; q < NPOS; ++q) ws[h][q] = w * pow2_bias(q * BITS);
  }
  if constexpr (BITS == 4) {
    // word 2k + hh, nibble n: channel 16k + 4(n>>1) + 2hh + (n&1); nibbles
    // 4..7 are read from word >> 16 at the positions of nibbles 0..3.
    const uint4 v = *reinterpret_cast<const uint4*>(cw);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int k = k4 >> 1, hh = k4 & 1;
      const uint32_t w16 = w[k4] >> 16;
      const float* wq = ws[NW == 1 ? 0 : k];
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const uint32_t m = 0xFu << (4 * n);
        const int ch = 16 * k + 4 * (n >> 1) + 2 * hh + (n & 1);
        acc[ch] = fmaf(wq[n], __uint_as_float(w[k4] & m), acc[ch]);
        acc[ch + 8] = fmaf(wq[n], __uint_as_float(w16 & m), acc[ch + 8]);
      }
    }
  } else {
    // word k: field f (channel 16k + f) at bits 2f; fields 8..15 are read from
    // word >> 16 at the positions of fields 0..7.
    const uint2 v = *reinterpret_cast<const uint2*>(cw);
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w16 = w[k] >> 16;
      const float* wq = ws[NW == 1 ? 0 : k];
#pragma unroll
      for (int f = 0; f < 8; ++f) {
        const uint32_t m = 3u << (2 * f);
        acc[16 * k + f] = fmaf(wq[f], __uint_as_float(w[k] & m), acc[16 * k + f]);
        acc[16 * k + 8 + f] = fmaf(wq[f], __uint_as_float(w16 & m), acc[16 * k + 8 + f]);
      }
    }
  }
}

// Components of a chain, unrolled at compile time: [own residual, ..., anchor].
template <class SP, int C = 0>
__device__ __forceinline__ void score_comps(const unsigned char* st, int j, int slice,
                                            const QLimbs& ql, float& part, float& kap) {
  if constexpr (C < SP::NC) {
    const float d = kdot<SP::D, SP::bits(C), SP::group(C)>(st + SP::codes_off(0, C),
                                                           st + SP::meta_off(0, C), j, slice, ql);
    part = fmaf(kap, d, part);
    if constexpr (SP::has_alpha(C))
      kap *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(st + SP::alpha_off(0, C))[j]);
    score_comps<SP, C + 1>(st, j, slice, ql, part, kap);
  }
}

template <class SP, int C = 0>
__device__ __forceinline__ void value_comps(const unsigned char* st, int j, int slice, float kap,
                                            float (&acc)[32], float (&cst)[2],
                                            uint32_t& range_err) {
  if constexpr (C < SP::NC) {
    vacc<SP::D, SP::bits(C), SP::group(C)>(st + SP::codes_off(1, C), st + SP::meta_off(1, C), j,
                                           slice, kap, acc, cst, range_err);
    if constexpr (SP::has_alpha(C))
      kap *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(st + SP::alpha_off(1, C))[j]);
    value_comps<SP, C + 1>(st, j, slice, kap, acc, cst, range_err);
  }
}

// Final value of the accumulators: undo the weight and subnormal scales and
// add the z~ terms of each 16-channel half.
__device__ __forceinline__ void finish_values(float (&acc)[32], const float (&cst)[2]) {
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) acc[ch] = fmaf(acc[ch], kValueUnscale, cst[ch / 16]);
}

// Token range of this CTA's split.
struct Range {
  int t_begin, t_end, nchunks;
};

__device__ __forceinline__ Range split_range(int n, int split, int cps, int tc) {
  Range r;
  r.t_begin = split * cps * tc;
  r.t_end = min(n, r.t_begin + cps * tc);
  r.nchunks = r.t_end > r.t_begin ? (r.t_end - r.t_begin + tc - 1) / tc : 0;
  return r;
}

// Producer loop (one lane): waits for a free stage, then issues the chunk's
// copies.
template <int S_MAX, typename Bytes, typename Issue>
__device__ __forceinline__ int produce(int nchunks, int S, uint64_t* full, uint64_t* empty,
                                       uint32_t* err, volatile int* abort_flag, Bytes bytes,
                                       Issue issue) {
  int issued = 0;
  for (int i = 0; i < nchunks; ++i) {
    const int s = i % S;
    if (i >= S) {
      if (!mbar_wait(&empty[s], ((i / S) - 1) & 1, err)) {
        *abort_flag = 1;
        break;
      }
    }
    if (*abort_flag) break;
    mbar_arrive_expect_tx(&full[s], bytes(i));
    issue(i, s);
    ++issued;
  }
  return issued;
}

// After an abort: wait (bounded) for every stage's most recent copies.
__device__ __forceinline__ void drain(int issued, int S, uint64_t* full, uint32_t* err) {
  for (int k = issued - S < 0 ? 0 : issued - S; k < issued; ++k)
    (void)mbar_wait(&full[k % S], (k / S) & 1, err);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Compressed decode.  Every warp consumes every stage; the warp that releases
// a stage last (a shared-memory counter, no waiting) issues that stage's
// refill with the chunk S ahead.
template <class SP>
__global__ void __launch_bounds__(kCThreads, kCMinCtas)
    decode_fast_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int D = SP::D, NC = SP::NC, TC = SP::TC;
  constexpr int P = D / 32, TPW = 32 / P, TPC = kCWarps * TPW, TT = TC / TPC;
  constexpr int NSLOT = kCWarps * TPW;
  static_assert(TT >= 1 && TT * TPC == TC, "chunk must be a multiple of the tokens per pass");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t full_bar[kMaxRing];
  __shared__ uint32_t s_release[kMaxRing];
  __shared__ float svec[D];
  __shared__ float sred[kCThreads / 32];
  __shared__ volatile int s_abort;
  __shared__ int s_issued;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int slice = lane % P, tw = lane / P;
  const int split = blockIdx.x, bhi = blockIdx.y;
  const int S = p.stages;
  const int n = seq_len_of(p.seq_lens, bhi / p.heads, p.max_seq_len, p.err);
  const Range R = split_range(n, split, p.chunks_per_split, TC);
  static_assert(TC == kBlock, "a decode stage is one storage record per component");

  // Copies of chunk i into stage s (one lane): one record per component.
  auto issue = [&](int i, int s) {
    const int t0 = R.t_begin + i * TC;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&full_bar[s], SP::stage_bytes());
    unsigned char* st = smem + static_cast<size_t>(s) * SP::stage_bytes();
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      const Comp* cs = side == 0 ? p.k : p.v;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        bulk_copy_g2s(st + SP::codes_off(side, c), comp_record(cs[c], bhi, p.nblk, t0),
                      SP::comp_bytes(c), &full_bar[s]);
    }
  };

  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      s_release[s] = 0u;
    }
    fence_barrier_init();
    s_abort = 0;
    const int first = min(S, R.nchunks);
    for (int i = 0; i < first; ++i) issue(i, i);
    s_issued = first;
  }
  // q' = H q * softmax scale * log2 e, rotated in registers by the P lanes of
  // each token slot (every slot holds the same query), then its fixed-point
  // scale from max |q'|.
  float qv[32];
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + static_cast<size_t>(bhi) * D + slice * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = src[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
        qv[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  }
  fwht_lanes<D>(qv, slice);
  const float qscale = p.rot_scale * p.scale_log2;
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    qv[i] *= qscale;
    amax = fmaxf(amax, fabsf(qv[i]));
  }
#pragma unroll
  for (int off = P / 2; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sigma = amax > 0.0f ? amax / 32639.0f : 1.0f;
  QLimbs ql;
  build_limbs(qv, 1.0f / sigma, ql);
  __syncthreads();   // barrier initialisation is visible to every warp
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
  float cst[2] = {0.0f, 0.0f};
  uint32_t range_err = 0u;
  float m = kNegInf, l = 0.0f;

  for (int i = 0; i < R.nchunks; ++i) {
    const int s = i % S;
    if (!mbar_wait(&full_bar[s], (i / S) & 1, p.err)) s_abort = 1;
    if (s_abort) break;
    const unsigned char* st = smem + static_cast<size_t>(s) * SP::stage_bytes();
    const int nt = min(TC, R.t_end - (R.t_begin + i * TC));
    float sc[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const int j = tt * TPC + warp * TPW + tw;
      float part = 0.0f, kap = 1.0f;
      score_comps<SP>(st, j, slice, ql, part, kap);
#pragma unroll
      for (int off = P / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      sc[tt] = (j < nt) ? part * sigma : kNegInf;
    }
    float mc = sc[0];
#pragma unroll
    for (int tt = 1; tt < TT; ++tt) mc = fmaxf(mc, sc[tt]);
    if (mc > m) {
      const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - mc);
      l *= f;
      cst[0] *= f;
      cst[1] *= f;
#pragma unroll
      for (int k = 0; k < 32; ++k) acc[k] *= f;
      m = mc;
    }
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const int j = tt * TPC + warp * TPW + tw;
      if (sc[tt] == kNegInf) continue;
      const float pt = fast_exp2(sc[tt] - m);
      l += pt;
      value_comps<SP>(st, j, slice, pt, acc, cst, range_err);
    }
    // Release the stage; the last warp to do so refills it.
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const uint32_t r = atomicAdd(&s_release[s], 1u);
      if (r % kCWarps == kCWarps - 1 && i + S < R.nchunks && !s_abort) {
        __threadfence_block();
        issue(i + S, s);
        atomicAdd(&s_issued, 1);
      }
    }
  }
  finish_values(acc, cst);
  if (range_err) atomicOr(p.err, kErrRange);
  if (s_abort) {
    m = kNegInf;
    l = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) acc[k] = 0.0f;
  }
  __syncthreads();
  if (s_abort && t == 0) drain(s_issued, S, full_bar, p.err);
  __syncthreads();
  finish_split<D, kCThreads, NSLOT, true>(m, l, acc, slice, warp * TPW + tw,
                                          reinterpret_cast<float*>(smem), bhi, split, p.splits,
                                          p.partials, p.counters, p.q, p.kcur, p.vcur,
                                          p.scale_log2, p.rot_scale, p.out, svec, sred);
}

// ---------------------------------------------------------------- BF16 --

template <int D>
__host__ __device__ constexpr int bf16_tc() { return D == 64 ? 128 : 64; }

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    decode_bf16_fast_kernel(const __grid_constant__ DecodeBf16Params p) {
  constexpr int TC = bf16_tc<D>();
  constexpr int P = D / 32, TPW = 32 / P, TPC = kWarps * TPW, TT = TC / TPC;
  constexpr int NSLOT = kWarps * TPW;
  constexpr uint32_t ROW = D * 2;
  constexpr uint32_t STAGE = 2 * TC * ROW;
  static_assert(TT >= 1 && TT * TPC == TC, "chunk must be a multiple of the tokens per pass");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t full_bar[kMaxRing], empty_bar[kMaxRing];
  __shared__ float svec[D];
  __shared__ float sred[kThreads / 32];
  __shared__ volatile int s_abort;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const bool producer = warp == kWarps;
  const int slice = lane % P, tw = lane / P;
  const int split = blockIdx.x, bhi = blockIdx.y;
  const int S = p.stages;
  const int n = seq_len_of(p.seq_lens, bhi / p.heads, p.max_seq_len, p.err);
  const Range R = split_range(n, split, p.chunks_per_split, TC);
  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kWarps);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  __syncthreads();
  float m = kNegInf, l = 0.0f;
  float acc[32];
  int slot = -1;
  if (producer) {
    if (lane == 0) {
      const size_t row0 = static_cast<size_t>(bhi) * p.tstride;
      auto bytes = [&](int i) -> uint32_t {
        return 2u * static_cast<uint32_t>(min(TC, R.t_end - (R.t_begin + i * TC))) * ROW;
      };
      auto issue = [&](int i, int s) {
        const int t0 = R.t_begin + i * TC;
        const uint32_t nt = static_cast<uint32_t>(min(TC, R.t_end - t0));
        unsigned char* st = smem + static_cast<size_t>(s) * STAGE;
        bulk_copy_g2s(st, p.k + (row0 + t0) * D, nt * ROW, &full_bar[s]);
        bulk_copy_g2s(st + TC * ROW, p.v + (row0 + t0) * D, nt * ROW, &full_bar[s]);
      };
      const int issued =
          produce<kMaxRing>(R.nchunks, S, full_bar, empty_bar, p.err, &s_abort, bytes, issue);
      if (s_abort) drain(issued, S, full_bar, p.err);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
  } else {
    slot = warp * TPW + tw;
    float2 q2[16];
    {
      const uint16_t* qr = p.q + static_cast<size_t>(bhi) * D + slice * 32;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        q2[i] = make_float2(bf16_bits_to_f32(qr[2 * i]) * p.scale_log2,
                            bf16_bits_to_f32(qr[2 * i + 1]) * p.scale_log2);
    }
    float2 acc2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc2[i] = make_float2(0.0f, 0.0f);
    for (int i = 0; i < R.nchunks; ++i) {
      const int s = i % S;
      if (!mbar_wait(&full_bar[s], (i / S) & 1, p.err)) s_abort = 1;
      if (s_abort) break;
      const unsigned char* st = smem + static_cast<size_t>(s) * STAGE;
      const int nt = min(TC, R.t_end - (R.t_begin + i * TC));
      float sc[TT];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const int j = tt * TPC + warp * TPW + tw;
        const uint4* kr = reinterpret_cast<const uint4*>(st + j * ROW + slice * 64);
        float2 part2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const uint4 v = kr[i4];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            part2 = __ffma2_rn(q2[i4 * 4 + e],
                               make_float2(__uint_as_float(w[e] << 16),
                                           __uint_as_float(w[e] & 0xFFFF0000u)),
                               part2);
        }
        float part = part2.x + part2.y;
#pragma unroll
        for (int off = P / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        sc[tt] = (j < nt) ? part : kNegInf;
      }
      float mc = sc[0];
#pragma unroll
      for (int tt = 1; tt < TT; ++tt) mc = fmaxf(mc, sc[tt]);
      if (mc > m) {
        const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - mc);
        const float2 f2 = make_float2(f, f);
        l *= f;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc2[k] = __fmul2_rn(acc2[k], f2);
        m = mc;
      }
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const int j = tt * TPC + warp * TPW + tw;
        if (sc[tt] == kNegInf) continue;
        const float pt = fast_exp2(sc[tt] - m);
        l += pt;
        const float2 p2 = make_float2(pt, pt);
        const uint4* vr = reinterpret_cast<const uint4*>(st + TC * ROW + j * ROW + slice * 64);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const uint4 v = vr[i4];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            acc2[i4 * 4 + e] = __ffma2_rn(p2,
                                          make_float2(__uint_as_float(w[e] << 16),
                                                      __uint_as_float(w[e] & 0xFFFF0000u)),
                                          acc2[i4 * 4 + e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      acc[2 * i] = acc2[i].x;
      acc[2 * i + 1] = acc2[i].y;
    }
    if (s_abort) {
      m = kNegInf;
      l = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
    }
  }
  __syncthreads();
  finish_split<D, kThreads, NSLOT, false>(m, l, acc, slice, slot, reinterpret_cast<float*>(smem),
                                          bhi, split, p.splits, p.partials, p.counters, p.q,
                                          p.kcur, p.vcur, p.scale_log2, 1.0f, p.out, svec, sred);
}

template <typename K>
cudaError_t prep(K kernel, size_t dyn, int* occ, int threads = kThreads) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(dyn));
  if (e != cudaSuccess) return e;
  if (occ != nullptr)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kernel, threads, dyn);
  return e;
}

// merge scratch of a kernel with `warps` compute warps: NSLOT*(D+2) floats
template <int D>
constexpr size_t scratch_floats(int warps = kWarps) {
  return static_cast<size_t>(warps * (32 / (D / 32))) * (D + 2);
}

template <class SP>
size_t dyn_bytes(int stages) {
  const size_t ring = static_cast<size_t>(stages) * SP::stage_bytes();
  size_t scr = scratch_floats<SP::D>(kCWarps) * sizeof(float);
  if (scr < kMergeScratch) scr = kMergeScratch;
  return ring > scr ? ring : scr;
}

// Host-side description of one compiled layout.
struct FastEntry {
  int D, NC, RB, RG, AB, AG;
  uint32_t stage_bytes;
  cudaError_t (*launch)(const DecodeParams&, cudaStream_t);
  cudaError_t (*occupancy)(int stages, int* occ);
};

template <class SP>
cudaError_t launch_spec(const DecodeParams& p, cudaStream_t s) {
  const size_t dyn = dyn_bytes<SP>(p.stages);
  cudaError_t e = prep(decode_fast_kernel<SP>, dyn, nullptr, kCThreads);
  if (e != cudaSuccess) return e;
  decode_fast_kernel<SP><<<dim3(p.splits, p.bh), kCThreads, dyn, s>>>(p);
  return cudaGetLastError();
}

template <class SP>
cudaError_t occ_spec(int stages, int* occ) {
  return prep(decode_fast_kernel<SP>, dyn_bytes<SP>(stages), occ, kCThreads);
}

#define RQ_FAST(D, NC, RB, RG, AB, AG)                                                        \
  FastEntry{D,  NC, RB, RG, AB, AG, Spec<D, NC, RB, RG, AB, AG>::stage_bytes(),              \
            &launch_spec<Spec<D, NC, RB, RG, AB, AG>>, &occ_spec<Spec<D, NC, RB, RG, AB, AG>>}

const FastEntry kFast[] = {
    // anchor loop alone
    RQ_FAST(128, 1, 2, 32, 4, 32), RQ_FAST(128, 1, 2, 64, 4, 64), RQ_FAST(128, 1, 2, 32, 2, 32),
    RQ_FAST(64, 1, 2, 32, 4, 32),
    // Last-loop: own residual + anchor
    RQ_FAST(128, 2, 2, 32, 4, 32), RQ_FAST(128, 2, 4, 32, 4, 32), RQ_FAST(128, 2, 2, 64, 4, 64),
    RQ_FAST(128, 2, 2, 16, 4, 32), RQ_FAST(128, 2, 2, 32, 2, 32), RQ_FAST(64, 2, 2, 32, 4, 32),
    // Next-loop chains (residuals share bits / group)
    RQ_FAST(128, 3, 2, 64, 4, 64), RQ_FAST(128, 4, 2, 64, 4, 64), RQ_FAST(128, 5, 2, 64, 4, 64),
    RQ_FAST(128, 6, 2, 64, 4, 64), RQ_FAST(128, 7, 2, 64, 4, 64), RQ_FAST(128, 8, 2, 64, 4, 64),
    RQ_FAST(128, 3, 2, 32, 4, 32), RQ_FAST(128, 4, 2, 32, 4, 32),
};

const FastEntry* find_fast(const DecodeParams& p, int D) {
  const int NC = p.ncomp;
  for (const FastEntry& f : kFast) {
    if (f.D != D || f.NC != NC) continue;
    bool ok = p.k[NC - 1].bits == f.AB && p.k[NC - 1].group == f.AG;
    for (int c = 0; c + 1 < NC; ++c) ok = ok && p.k[c].bits == f.RB && p.k[c].group == f.RG;
    // a stage is exactly one record per component and side
    uint32_t rec = 0;
    for (int c = 0; c < NC; ++c) rec += p.k[c].rec_bytes + p.v[c].rec_bytes;
    ok = ok && rec == f.stage_bytes;
    if (ok) return &f;
  }
  return nullptr;
}

template <int D>
cudaError_t launch_bf16_t(const DecodeBf16Params& p, cudaStream_t s) {
  const size_t ring = static_cast<size_t>(p.stages) * (2 * bf16_tc<D>() * D * 2);
  size_t scr = scratch_floats<D>() * sizeof(float);
  if (scr < kMergeScratch) scr = kMergeScratch;
  const size_t dyn = ring > scr ? ring : scr;
  cudaError_t e = prep(decode_bf16_fast_kernel<D>, dyn, nullptr);
  if (e != cudaSuccess) return e;
  decode_bf16_fast_kernel<D><<<dim3(p.splits, p.bh), kThreads, dyn, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

// ---- host interface (rq_internal.cuh) ----

bool fast_decode_plan(const DecodeParams& p, int D, size_t ring_budget, int max_stages,
                      int* stages, int* ctas_per_sm) {
  const FastEntry* f = find_fast(p, D);
  if (f == nullptr) return false;
  (void)ring_budget;
  int s = static_cast<int>(kCRingBudget / f->stage_bytes);
  if (s > max_stages) s = max_stages;
  if (s > kMaxRing) s = kMaxRing;
  if (s < 2) s = 2;
  if (static_cast<size_t>(s) * f->stage_bytes > 220 * 1024) return false;
  int occ = 0;
  if (f->occupancy(s, &occ) != cudaSuccess || occ < 1) return false;
  *stages = s;
  *ctas_per_sm = occ;
  return true;
}

cudaError_t launch_decode_fast(const DecodeParams& p, int D, cudaStream_t s) {
  const FastEntry* f = find_fast(p, D);
  if (f == nullptr) return cudaErrorInvalidValue;
  return f->launch(p, s);
}

uint32_t bf16_stage_bytes(int D) {
  return D == 64 ? 2u * bf16_tc<64>() * 64 * 2 : 2u * bf16_tc<128>() * 128 * 2;
}
int bf16_chunk(int D) { return D == 64 ? bf16_tc<64>() : bf16_tc<128>(); }
int fast_chunk() { return kCChunk; }

cudaError_t bf16_occupancy(int D, int stages, int* occ) {
  const size_t ring = static_cast<size_t>(stages) * bf16_stage_bytes(D);
  if (D == 64) {
    const size_t scr = scratch_floats<64>() * sizeof(float);
    return prep(decode_bf16_fast_kernel<64>, ring > scr ? ring : scr, occ);
  }
  const size_t scr = scratch_floats<128>() * sizeof(float);
  return prep(decode_bf16_fast_kernel<128>, ring > scr ? ring : scr, occ);
}

cudaError_t launch_decode_bf16(const DecodeBf16Params& p, int D, cudaStream_t s) {
  if (D == 64) return launch_bf16_t<64>(p, s);
  if (D == 128) return launch_bf16_t<128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace rq
