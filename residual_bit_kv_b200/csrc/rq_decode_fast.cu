// rq_decode_fast.cu -- split-K decode attention for the packed ResidualQuant
// cache with compile-time component layouts, and for the uncompressed BF16
// baseline.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// Compressed kernel: a CTA of 4 warps streams one (batch*head, split) token
// range in stages of two 32-token storage records per component and side
// (one bulk asynchronous copy each) through an S-stage shared-memory
// ring.  Every warp consumes every stage; the warp that releases a stage last
// issues its refill, S stages ahead.
//
// Scores [RQ §4.1, App. G.2]: q' = H q (pre-scaled by softmax scale and
// log2 e) is held as 16-bit fixed point, q' ~= sigma * (256 h + l) with
// int8 limbs h, l, so q'.codes over a group is two integer dot products
// (dp4a) of the unpacked code bytes with the limbs; the score of a token is
// sigma * sum_c kappa_c (s~_c * dot_c + z~_c * sum q~), kappa the product of
// the LS coefficients along the reference chain.
// Values: a code masked out of its word (all other bits zero) is the exact
// fp32 subnormal c * 2^(p-149), p its bit position; packed fp32 FMAs with
// weights p_t * kappa * s~ * 2^(92-p) accumulate p_t * kappa * s~ * c * 2^-57
// per channel, the offsets z~ going to separate accumulators.  Accumulation
// is in the rotated domain; H^T is applied once in the merge.
#include <type_traits>

#include "rq_decode_common.cuh"

namespace rq {
namespace {

// Shared-memory atomic add returning the old value (one lane; no warp
// aggregation).
__device__ __forceinline__ uint32_t atom_add_shared(uint32_t* a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(a)), "r"(v)
               : "memory");
  return old;
}

constexpr int kWarps = 8;                      // BF16 kernel: compute warps per CTA
constexpr int kThreads = (kWarps + 1) * 32;    // + producer warp
constexpr int kMaxRing = 4;                    // BF16 kernel ring

constexpr int kCWarps = 4;                     // compressed kernel: warps per CTA
constexpr int kCThreads = kCWarps * 32;
constexpr int kCMaxRing = 8;                   // compressed kernel ring
constexpr int kCMinCtas = 5;                   // register target: CTAs per SM
constexpr size_t kCRingBudget = 43 * 1024;     // stage ring per CTA (5 CTAs per SM)
constexpr size_t kMergeScratch = 3 * 1024 * sizeof(float);   // split headers, up to 1024 splits

// Compile-time layout of one stage: for side K then V, component c occupies
// RPS = 2 consecutive records (64 tokens, one copy); a record is
// [codes[32][wpr] | meta[32][gpr] | alpha[32]].
template <int D_, int NC_, int RB_, int RG_, int AB_, int AG_, int M16_ = 0, int MU_ = 0>
struct Spec {
  // M16: 16-bit metadata per group; MU: the residual loops carry fixed means [RQ App. G.2]
  static constexpr int D = D_, NC = NC_, RPS = 2, TC = kBlock * RPS, M16 = M16_, MU = MU_;
  __host__ __device__ static constexpr int bits(int c) { return c == NC_ - 1 ? AB_ : RB_; }
  __host__ __device__ static constexpr int group(int c) { return c == NC_ - 1 ? AG_ : RG_; }
  __host__ __device__ static constexpr bool has_alpha(int c) { return c != NC_ - 1; }
  __host__ __device__ static constexpr int wpr(int c) { return D_ * bits(c) / 32; }
  __host__ __device__ static constexpr int gpr(int c) { return D_ / group(c); }
  __host__ __device__ static constexpr uint32_t rec_bytes(int c) {
    return kBlock * (wpr(c) * 4 + gpr(c) * (M16_ ? 2 : 4) + (has_alpha(c) ? 2 : 0));
  }
  __host__ __device__ static constexpr uint32_t comp_bytes(int c) { return RPS * rec_bytes(c); }
  __host__ __device__ static constexpr uint32_t side_bytes() {
    uint32_t s = 0;
    for (int c = 0; c < NC_; ++c) s += comp_bytes(c);
    return s;
  }
  __host__ __device__ static constexpr uint32_t stage_bytes() { return 2 * side_bytes(); }
  __host__ __device__ static constexpr uint32_t comp_off(int side, int c) {
    uint32_t o = side * side_bytes();
    for (int k = 0; k < c; ++k) o += comp_bytes(k);
    return o;
  }
  // Record of component c (side) holding stage token j.
  __device__ static const unsigned char* rec(const unsigned char* st, int side, int c, int j) {
    return st + comp_off(side, c) + (RPS == 1 ? 0 : (j / kBlock) * rec_bytes(c));
  }
};

// Offsets inside a record of a component with these parameters (M16: 16-bit
// metadata per group).
template <int D, int BITS, int G, int M16 = 0>
struct RecGeom {
  enum : uint32_t {
    WPR = D * BITS / 32,
    GPR = D / G,
    META = kBlock * WPR * 4,
    ALPHA = META + kBlock * GPR * (M16 ? 2 : 4),
  };
};

// Scale and offset of this lane's group(s) at record token jl: [0] channels
// 0-15 (or the whole slice when g >= 32), [1] channels 16-31 (g = 16).
template <int D, int BITS, int G, int M16>
__device__ __forceinline__ void group_meta(const unsigned char* rec, int jl, int slice,
                                           float (&s)[2], float (&z)[2]) {
  using RG = RecGeom<D, BITS, G, M16>;
  if constexpr (M16) {
    const uint16_t* mr = reinterpret_cast<const uint16_t*>(rec + RG::META) + jl * RG::GPR;
    if constexpr (G >= 32) {
      const uint32_t h = mr[(slice * 32) / G];
      s[0] = s[1] = m16_scale_value(h & 0xFFu);
      z[0] = z[1] = m16_offset(h, s[0]);
    } else {
      const uint32_t hh = *reinterpret_cast<const uint32_t*>(mr + slice * 2);
      s[0] = m16_scale_value(hh & 0xFFu);
      z[0] = m16_offset(hh & 0xFFFFu, s[0]);
      s[1] = m16_scale_value((hh >> 16) & 0xFFu);
      z[1] = m16_offset(hh >> 16, s[1]);
    }
  } else {
    const uint32_t* mr = reinterpret_cast<const uint32_t*>(rec + RG::META) + jl * RG::GPR;
    if constexpr (G >= 32) {
      unpack_meta(mr[(slice * 32) / G], s[0], z[0]);
      s[1] = s[0];
      z[1] = z[0];
    } else {
      const uint2 mw = *reinterpret_cast<const uint2*>(mr + slice * 2);
      unpack_meta(mw.x, s[0], z[0]);
      unpack_meta(mw.y, s[1], z[1]);
    }
  }
}

// Fixed-point rotated query of one lane's 32 channels as int8 limb bytes in
// the quad order of the unpacked codes: quad (k, s) holds channels
// 16k + s + {0, 4, 8, 12} (the same for 2-bit and 4-bit codes).
struct QLimbs {
  int h[2][4], l[2][4];
  float sq[2];   // sum of q~ over channels 0-15 / 16-31
};

// q~ . D(c) over one lane's 32 channels of record token jl of a component,
// in sigma units: sum over group parts of s~ * (q~ . codes) + z~ * (sum q~).
template <int D, int BITS, int G, int M16>
__device__ __forceinline__ float kdot(const unsigned char* rec, int jl, int slice,
                                      const QLimbs& ql) {
  using RG = RecGeom<D, BITS, G, M16>;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(rec) + jl * RG::WPR + slice * BITS;
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
  float sm[2], zm[2];
  group_meta<D, BITS, G, M16>(rec, jl, slice, sm, zm);
  if constexpr (G >= 32) {
    return sm[0] * static_cast<float>((ah[0] + ah[1]) * 256 + (al[0] + al[1])) +
           zm[0] * (ql.sq[0] + ql.sq[1]);
  } else {
    return sm[0] * static_cast<float>(ah[0] * 256 + al[0]) + zm[0] * ql.sq[0] +
           (sm[1] * static_cast<float>(ah[1] * 256 + al[1]) + zm[1] * ql.sq[1]);
  }
}

// Value accumulators of one lane: channel pairs (2i, 2i+1) of its 32-channel
// slice as packed fp32 (acc[i]); z~ terms per 16-channel half (cst[0], cst[1])
// and for groups spanning the whole slice (cst[2]).
struct VAcc {
  float2 acc[16];
  float cst[3];
  float mw[8];   // fixed means: sum of p_t * kappa_c per residual component (MU layouts)
};

// Weights w * 2^(92 - p), p <= 14: finite for w < 2^36, and products stay
// normal down to w * c = 2^-69.
constexpr int kPosBias = 92;
constexpr float kValueUnscale = 144115188075855872.0f;   // 2^(149 - kPosBias) = 2^57

__device__ __forceinline__ float pow2i(int e) {
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

__device__ __forceinline__ float2 masked_pair(uint32_t w, uint32_t ma, uint32_t mb) {
  return make_float2(__uint_as_float(w & ma), __uint_as_float(w & mb));
}

// acc += pk * D(c) over one lane's 32 channels of record token jl (codes
// part; the z~ offsets go to cst).  A channel pair shares a word, and the
// code positions (pa, pb) of the pair fix its weight pair
// {w 2^(92-pa), w 2^(92-pb)}, w = pk * s~:
//   b = 2: word k holds channels 16k + 2i, +1 at bits 4i, 4i+2 (i < 4), and
//          channels 16k + 8 + 2i, +1 at the same bits of word >> 16;
//   b = 4: word 2k + hh holds channels 16k + 2hh, +1 at bits 0, 4 and
//          16k + 4 + 2hh, +1 at bits 8, 12; word >> 16 gives channels + 8.
template <int D, int BITS, int G, int M16>
__device__ __forceinline__ void vacc(const unsigned char* rec, int jl, int slice, float pk,
                                     VAcc& va) {
  using RG = RecGeom<D, BITS, G, M16>;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(rec) + jl * RG::WPR + slice * BITS;
  constexpr int NW = G >= 32 ? 1 : 2;   // weights per lane (16-channel halves for g = 16)
  float sc[2], zc[2];
  group_meta<D, BITS, G, M16>(rec, jl, slice, sc, zc);
  if constexpr (NW == 1) {
    va.cst[2] = fmaf(pk, zc[0], va.cst[2]);
  } else {
    va.cst[0] = fmaf(pk, zc[0], va.cst[0]);
    va.cst[1] = fmaf(pk, zc[1], va.cst[1]);
  }
  constexpr int NP = BITS == 2 ? 4 : 2;   // distinct weight pairs
  float2 wp[NW][NP];
#pragma unroll
  for (int h = 0; h < NW; ++h) {
    const float w = pk * sc[h];
    const float2 ww = make_float2(w, w);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int pa = BITS == 2 ? 4 * i : 8 * i;
      const int pb = pa + BITS;
      wp[h][i] = __fmul2_rn(ww, make_float2(pow2i(kPosBias - pa), pow2i(kPosBias - pb)));
    }
  }
  if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(cw);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int k = k4 >> 1, hh = k4 & 1;
      const uint32_t w16 = w[k4] >> 16;
      const float2* wq = wp[NW == 1 ? 0 : k];
      float2* a = va.acc + 8 * k + hh;
      a[0] = __ffma2_rn(wq[0], masked_pair(w[k4], 0xFu, 0xF0u), a[0]);
      a[2] = __ffma2_rn(wq[1], masked_pair(w[k4], 0xF00u, 0xF000u), a[2]);
      a[4] = __ffma2_rn(wq[0], masked_pair(w16, 0xFu, 0xF0u), a[4]);
      a[6] = __ffma2_rn(wq[1], masked_pair(w16, 0xF00u, 0xF000u), a[6]);
    }
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(cw);
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w16 = w[k] >> 16;
      const float2* wq = wp[NW == 1 ? 0 : k];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t ma = 3u << (4 * i), mb = 3u << (4 * i + 2);
        va.acc[8 * k + i] = __ffma2_rn(wq[i], masked_pair(w[k], ma, mb), va.acc[8 * k + i]);
        va.acc[8 * k + 4 + i] =
            __ffma2_rn(wq[i], masked_pair(w16, ma, mb), va.acc[8 * k + 4 + i]);
      }
    }
  }
}

// Components of a chain, unrolled at compile time: [own residual, ..., anchor].
// REC is the stage record (compile-time), jl the token inside it.
template <class SP, int REC, int C = 0>
__device__ __forceinline__ void score_comps(const unsigned char* st, int rl, int jl, int slice,
                                            const QLimbs& ql, const float* qmu, float& part,
                                            float& kap) {
  if constexpr (C < SP::NC) {
    using RG = RecGeom<SP::D, SP::bits(C), SP::group(C), SP::M16>;
    const unsigned char* rec = st + SP::comp_off(0, C) + (REC + rl) * SP::rec_bytes(C);
    const float d = kdot<SP::D, SP::bits(C), SP::group(C), SP::M16>(rec, jl, slice, ql);
    part = fmaf(kap, d, part);
    // the mean's share: kappa * (q~ . mu) over this lane's channels
    if constexpr (SP::MU && SP::has_alpha(C)) part = fmaf(kap, qmu[C], part);
    if constexpr (SP::has_alpha(C))
      kap *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(rec + RG::ALPHA)[jl]);
    score_comps<SP, REC, C + 1>(st, rl, jl, slice, ql, qmu, part, kap);
  }
}

template <class SP, int REC, int C = 0>
__device__ __forceinline__ void value_comps(const unsigned char* st, int rl, int jl, int slice,
                                            float kap, VAcc& va) {
  if constexpr (C < SP::NC) {
    using RG = RecGeom<SP::D, SP::bits(C), SP::group(C), SP::M16>;
    const unsigned char* rec = st + SP::comp_off(1, C) + (REC + rl) * SP::rec_bytes(C);
    vacc<SP::D, SP::bits(C), SP::group(C), SP::M16>(rec, jl, slice, kap, va);
    if constexpr (SP::MU && SP::has_alpha(C)) va.mw[C] += kap;
    if constexpr (SP::has_alpha(C))
      kap *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(rec + RG::ALPHA)[jl]);
    value_comps<SP, REC, C + 1>(st, rl, jl, slice, kap, va);
  }
}

// The TT tokens of one chunk held by this thread.  Token tt of the thread is
// stage token tt * TPC + jr: record tt * TPC / 32 + rl (rl = jr / 32, zero
// when a CTA pass is one record), row jl = jr % 32.  MASK: the chunk may end
// before TC tokens (nt < TC); full chunks skip the per-token tests.
template <class SP, int TT, int TPC, int P, bool MASK, int TTI = 0>
__device__ __forceinline__ void chunk_scores(const unsigned char* st, int jr, int rl, int jl,
                                             int slice, const QLimbs& ql, const float* qmu,
                                             float sigma, int nt, float (&sc)[TT]) {
  if constexpr (TTI < TT) {
    float part = 0.0f, kap = 1.0f;
    score_comps<SP, TTI * TPC / kBlock>(st, rl, jl, slice, ql, qmu, part, kap);
#pragma unroll
    for (int off = P / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    sc[TTI] = (!MASK || TTI * TPC + jr < nt) ? part * sigma : kNegInf;
    chunk_scores<SP, TT, TPC, P, MASK, TTI + 1>(st, jr, rl, jl, slice, ql, qmu, sigma, nt, sc);
  }
}

template <class SP, int TT, int TPC, bool MASK, int TTI = 0>
__device__ __forceinline__ void chunk_values(const unsigned char* st, int rl, int jl, int slice,
                                             const float (&sc)[TT], float m, float& l, VAcc& va) {
  if constexpr (TTI < TT) {
    if (!MASK || sc[TTI] != kNegInf) {
      const float pt = fast_exp2(sc[TTI] - m);
      l += pt;
      value_comps<SP, TTI * TPC / kBlock>(st, rl, jl, slice, pt, va);
    }
    chunk_values<SP, TT, TPC, MASK, TTI + 1>(st, rl, jl, slice, sc, m, l, va);
  }
}

template <int MU = 0, int NC = 1>
__device__ __forceinline__ void rescale(VAcc& va, float f) {
  const float2 ff = make_float2(f, f);
#pragma unroll
  for (int i = 0; i < 16; ++i) va.acc[i] = __fmul2_rn(va.acc[i], ff);
  va.cst[0] *= f;
  va.cst[1] *= f;
  va.cst[2] *= f;
  if constexpr (MU) {
#pragma unroll
    for (int c = 0; c + 1 < NC; ++c) va.mw[c] *= f;
  }
}

// Final per-channel values: undo the 2^-40 code scale and add the z~ terms.
// A weight past the scaled range (p_t * kappa * s~ >= 2^36) leaves an
// infinity or NaN here and is reported.
__device__ __forceinline__ void finish_values(const VAcc& va, float (&acc)[32],
                                              uint32_t& range_err) {
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float c = va.cst[i / 8] + va.cst[2];
    acc[2 * i] = fmaf(va.acc[i].x, kValueUnscale, c);
    acc[2 * i + 1] = fmaf(va.acc[i].y, kValueUnscale, c);
    finite = finite && isfinite(acc[2 * i]) && isfinite(acc[2 * i + 1]);
  }
  if (!finite) range_err = 1u;
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
  __shared__ uint64_t full_bar[kCMaxRing];
  __shared__ uint32_t s_release[kCMaxRing];
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

  // Copies of chunk i into stage s (one lane): RPS consecutive records per
  // component and side, one copy each.  Splits start at multiples of TC
  // tokens and rows hold a multiple of 64 tokens, so a stage never leaves
  // its row.
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
        bulk_copy_g2s(st + SP::comp_off(side, c), comp_record(cs[c], bhi, p.nblk, t0),
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
  // q' = H q * softmax scale * log2 e, one channel per thread (every split
  // of a row forms the same q'), its fixed-point scale sigma from max |q'|,
  // and the int8 limbs stored in the quad order each lane reads: channel
  // 32*sl + 16k + s + 4u goes to word 8*sl + 4k + s, byte u.
  __shared__ __align__(16) int s_limb[2][D / 4];
  __shared__ float s_sq[D / 16];
  __shared__ float s_amax[kCWarps];
  if (t < D) svec[t] = bf16_bits_to_f32(p.q[static_cast<size_t>(bhi) * D + t]);
  __syncthreads();
  const int qhead = bhi % p.heads;
  const float qscale =
      rotate_query<D>(svec, p.urot_k ? p.urot_k + static_cast<size_t>(qhead) * D * D : nullptr,
                      p.rot_scale) *
      p.scale_log2;
  const float qv = t < D ? svec[t] * qscale : 0.0f;
  float amax = fabsf(qv);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) s_amax[warp] = amax;
  __syncthreads();
  amax = s_amax[0];
#pragma unroll
  for (int w = 1; w < kCWarps; ++w) amax = fmaxf(amax, s_amax[w]);
  const float sigma = amax > 0.0f ? amax / 32639.0f : 1.0f;
  {
    const int qt = __float2int_rn(qv * (1.0f / sigma));   // |qt| <= 32639
    const int hi = (qt + 128) >> 8;
    float qs = static_cast<float>(qt);
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, off);
    if (t < D) {
      const int c = t & 31;
      const int byte = (t >> 5) * 32 + ((c >> 4) * 4 + (c & 3)) * 4 + ((c >> 2) & 3);
      reinterpret_cast<signed char*>(s_limb[0])[byte] = static_cast<signed char>(hi);
      reinterpret_cast<signed char*>(s_limb[1])[byte] = static_cast<signed char>(qt - 256 * hi);
      if ((c & 15) == 0) s_sq[t >> 4] = qs;
    }
  }
  __syncthreads();
  QLimbs ql;
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      ql.h[k][q4] = s_limb[0][slice * 8 + k * 4 + q4];
      ql.l[k][q4] = s_limb[1][slice * 8 + k * 4 + q4];
    }
  ql.sq[0] = s_sq[slice * 2];
  ql.sq[1] = s_sq[slice * 2 + 1];
  // Fixed means [RQ App. G.2]: q~ . mu_c over this lane's 32 channels, per
  // residual component of the K chain (one warp per slice).
  float qmu[SP::NC];
#pragma unroll
  for (int c = 0; c < SP::NC; ++c) qmu[c] = 0.0f;
  if constexpr (SP::MU) {
    __shared__ float s_qmu[SP::NC][kCWarps];
    const int head = bhi % p.k[0].heads;
#pragma unroll
    for (int c = 0; c + 1 < SP::NC; ++c) {
      const float* mu = p.k[c].mean;
      float v = (mu != nullptr && t < D) ? (qv * (1.0f / sigma)) * mu[head * D + t] : 0.0f;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) s_qmu[c][warp] = v;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c + 1 < SP::NC; ++c) qmu[c] = s_qmu[c][slice];
  }
  VAcc va;
#pragma unroll
  for (int i = 0; i < 16; ++i) va.acc[i] = make_float2(0.0f, 0.0f);
  va.cst[0] = va.cst[1] = va.cst[2] = 0.0f;
#pragma unroll
  for (int c = 0; c < 8; ++c) va.mw[c] = 0.0f;
  float m = kNegInf, l = 0.0f;

  // This thread's tokens: jr inside a CTA pass of TPC tokens.
  const int jr = warp * TPW + tw;
  const int rl = TPC == kBlock ? 0 : jr / kBlock;
  const int jl = jr % kBlock;
  auto chunk = [&](const unsigned char* st, auto mask_tag, int nt) {
    constexpr bool MASK = decltype(mask_tag)::value;
    float sc[TT];
    chunk_scores<SP, TT, TPC, P, MASK>(st, jr, rl, jl, slice, ql, qmu, sigma, nt, sc);
    float mc = sc[0];
#pragma unroll
    for (int tt = 1; tt < TT; ++tt) mc = fmaxf(mc, sc[tt]);
    if (mc > m) {
      const float f = (m == kNegInf) ? 0.0f : fast_exp2(m - mc);
      l *= f;
      rescale<SP::MU, SP::NC>(va, f);
      m = mc;
    }
    chunk_values<SP, TT, TPC, MASK>(st, rl, jl, slice, sc, m, l, va);
  };
  int s = 0;
  uint32_t phase = 0u;
  for (int i = 0; i < R.nchunks; ++i) {
    if (!mbar_wait(&full_bar[s], phase, p.err)) {
      s_abort = 1;   // this warp stops; the others stop at their own timeout
      break;
    }
    const unsigned char* st = smem + static_cast<size_t>(s) * SP::stage_bytes();
    const int nt = R.t_end - (R.t_begin + i * TC);
    if (nt >= TC)
      chunk(st, std::integral_constant<bool, false>{}, TC);
    else
      chunk(st, std::integral_constant<bool, true>{}, nt);
    // Release the stage; the last warp to do so refills it.
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const uint32_t r = atom_add_shared(&s_release[s], 1u);
      if (r % kCWarps == kCWarps - 1 && i + S < R.nchunks && !s_abort) {
        __threadfence_block();
        issue(i + S, s);
        atom_add_shared(reinterpret_cast<uint32_t*>(&s_issued), 1u);
      }
    }
    if (++s == S) {
      s = 0;
      phase ^= 1u;
    }
  }
  float acc[32];
  uint32_t range_err = 0u;
  finish_values(va, acc, range_err);
  if constexpr (SP::MU) {
    // sum_t p_t kappa_c mu_c over this lane's channels
    const int head = bhi % p.v[0].heads;
#pragma unroll
    for (int c = 0; c + 1 < SP::NC; ++c) {
      const float* mu = p.v[c].mean;
      if (mu == nullptr) continue;
      const float4* src = reinterpret_cast<const float4*>(mu + head * D + slice * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 e = src[i];
        acc[4 * i] = fmaf(va.mw[c], e.x, acc[4 * i]);
        acc[4 * i + 1] = fmaf(va.mw[c], e.y, acc[4 * i + 1]);
        acc[4 * i + 2] = fmaf(va.mw[c], e.z, acc[4 * i + 2]);
        acc[4 * i + 3] = fmaf(va.mw[c], e.w, acc[4 * i + 3]);
      }
    }
  }
  __syncthreads();   // every warp has left the loop: s_abort is settled
  const bool aborted = s_abort != 0;
  const bool range_bad = __syncthreads_or(range_err != 0u) != 0;
  if (range_err && !aborted) atomicOr(p.err, kErrRange);
  if (aborted) {
    m = kNegInf;
    l = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) acc[k] = 0.0f;
    if (t == 0) drain(s_issued, S, full_bar, p.err);
  }
  __syncthreads();
  finish_split<D, kCThreads, NSLOT, true>(m, l, acc, slice, warp * TPW + tw,
                                          reinterpret_cast<float*>(smem), bhi, split, p.splits,
                                          p.partials, p.counters, p.q, p.kcur, p.vcur,
                                          p.scale_log2, p.rot_scale, p.out, svec, sred,
                                          aborted || range_bad,
                                          p.urot_v ? p.urot_v + static_cast<size_t>(bhi % p.heads) *
                                                                    D * D
                                                   : nullptr);
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
  const bool aborted = __syncthreads_or(s_abort != 0) != 0;
  finish_split<D, kThreads, NSLOT, false>(m, l, acc, slice, slot, reinterpret_cast<float*>(smem),
                                          bhi, split, p.splits, p.partials, p.counters, p.q,
                                          p.kcur, p.vcur, p.scale_log2, 1.0f, p.out, svec, sred,
                                          aborted);
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

// merge scratch of a kernel with `warps` compute warps: NSLOT*(pitch+2) floats
template <int D>
constexpr size_t scratch_floats(int warps = kWarps) {
  return static_cast<size_t>(warps * (32 / (D / 32))) * (red_pitch<D>() + 2);
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
  int D, NC, RB, RG, AB, AG, M16, MU;
  uint32_t stage_bytes;
  int chunk;
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

#define RQ_FAST_X(D, NC, RB, RG, AB, AG, M, MU)                                                \
  FastEntry{D,  NC, RB, RG, AB, AG, M, MU, Spec<D, NC, RB, RG, AB, AG, M, MU>::stage_bytes(),  \
            Spec<D, NC, RB, RG, AB, AG, M, MU>::TC,                                          \
            &launch_spec<Spec<D, NC, RB, RG, AB, AG, M, MU>>,                                \
            &occ_spec<Spec<D, NC, RB, RG, AB, AG, M, MU>>}
#define RQ_FAST(D, NC, RB, RG, AB, AG) RQ_FAST_X(D, NC, RB, RG, AB, AG, 0, 0)
#define RQ_FAST16(D, NC, RB, RG, AB, AG) RQ_FAST_X(D, NC, RB, RG, AB, AG, 1, 0)
#define RQ_FAST_MU(D, NC, RB, RG, AB, AG) RQ_FAST_X(D, NC, RB, RG, AB, AG, 0, 1)

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
    // 16-bit metadata: anchor alone, Last-loop pairs, Next-loop chains
    RQ_FAST16(128, 1, 2, 32, 4, 32), RQ_FAST16(128, 2, 2, 32, 4, 32),
    RQ_FAST16(128, 2, 4, 32, 4, 32), RQ_FAST16(128, 2, 2, 16, 4, 32),
    RQ_FAST16(128, 3, 2, 32, 4, 32), RQ_FAST16(128, 4, 2, 32, 4, 32),
    RQ_FAST16(64, 1, 2, 32, 4, 32), RQ_FAST16(64, 2, 2, 32, 4, 32),
    // residual loops with fixed means: Last-loop pairs and Next-loop chains
    RQ_FAST_MU(128, 2, 2, 32, 4, 32), RQ_FAST_MU(128, 2, 4, 32, 4, 32),
    RQ_FAST_MU(128, 3, 2, 32, 4, 32), RQ_FAST_MU(128, 4, 2, 32, 4, 32),
    RQ_FAST_MU(64, 2, 2, 32, 4, 32),
};

const FastEntry* find_fast(const DecodeParams& p, int D) {
  const int NC = p.ncomp;
  for (const FastEntry& f : kFast) {
    const int mu = (p.k[0].mean != nullptr || p.v[0].mean != nullptr) ? 1 : 0;
    if (f.D != D || f.NC != NC || f.M16 != p.k[0].meta16 || f.MU != mu) continue;
    bool ok = p.k[NC - 1].bits == f.AB && p.k[NC - 1].group == f.AG;
    for (int c = 0; c + 1 < NC; ++c) ok = ok && p.k[c].bits == f.RB && p.k[c].group == f.RG;
    // a stage is exactly RPS records per component and side
    uint32_t rec = 0;
    for (int c = 0; c < NC; ++c) rec += p.k[c].rec_bytes + p.v[c].rec_bytes;
    ok = ok && rec * (f.chunk / kBlock) == f.stage_bytes;
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

bool fast_decode_plan(const DecodeParams& p, int D, int* stages, int* chunk, int* ctas_per_sm) {
  const FastEntry* f = find_fast(p, D);
  if (f == nullptr) return false;
  int s = static_cast<int>(kCRingBudget / f->stage_bytes);
  if (s > kCMaxRing) s = kCMaxRing;
  if (s < 2) s = 2;
  if (static_cast<size_t>(s) * f->stage_bytes > 220 * 1024) return false;
  int occ = 0;
  if (f->occupancy(s, &occ) != cudaSuccess || occ < 1) return false;
  *stages = s;
  *chunk = f->chunk;
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
