// rq_decode.cu -- generic split-K decode attention over the packed
// ResidualQuant cache: any chain of components with run-time bit widths and
// group sizes.  Layouts compiled into rq_decode_fast.cu take the
// warp-specialised kernel instead; this one covers every other layout.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// Work decomposition: one CTA (128 threads) per (batch*head, split); a split
// is a contiguous range of past tokens.  Each CTA streams its range in chunks
// of kChunk tokens (two 32-token storage records): thread 0 issues one bulk
// asynchronous copy per component and side (codes, metadata and LS
// coefficients of two consecutive records are contiguous) into an S-stage
// shared-memory ring, completing on a per-stage mbarrier; all
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
#include "rq_decode_common.cuh"

namespace rq {
namespace {

template <int D>
struct Geom {
  static constexpr int P = D / 32;            // lanes per token
  static constexpr int TPW = 32 / P;          // tokens per warp pass
  static constexpr int TPC = 4 * TPW;         // tokens per CTA pass
  static constexpr int TT = kChunk / TPC;     // tokens per thread per chunk
  static constexpr int NSLOT = kDecodeThreads / P;
};

// Per-component shared-memory layout of one pipeline stage: component c of
// side `side` occupies kChunk/kBlock consecutive records (one copy) starting
// at comp[side][c]; inside a record, codes start at 0, metadata at meta[..]
// and LS coefficients at alpha[..].
struct StageMap {
  uint32_t comp[2][RQ_MAX_LOOPS];
  uint32_t meta[2][RQ_MAX_LOOPS];
  uint32_t alpha[2][RQ_MAX_LOOPS];
  uint32_t bytes;
};

constexpr int kRecsPerStage = kChunk / kBlock;

__host__ __device__ inline void build_stage_map(const DecodeParams& p, int D,
                                                StageMap& m) {
  uint32_t off = 0;
  for (int side = 0; side < 2; ++side) {
    const Comp* cs = side == 0 ? p.k : p.v;
    for (int c = 0; c < p.ncomp; ++c) {
      m.comp[side][c] = off;
      m.meta[side][c] = kBlock * (D * cs[c].bits / 32) * 4;
      m.alpha[side][c] = m.meta[side][c] + kBlock * (D / cs[c].group) * (cs[c].meta16 ? 2 : 4);
      off += kRecsPerStage * cs[c].rec_bytes;
    }
  }
  m.bytes = off;
}

// Start of the record holding stage token j of component c.
__device__ __forceinline__ const unsigned char* stage_rec(const unsigned char* st,
                                                          const StageMap& m, const Comp& cp,
                                                          int side, int c, int j) {
  return st + m.comp[side][c] + (j / kBlock) * cp.rec_bytes;
}

// Scale and offset of this lane's group parts from one token's metadata row
// (fp16 pairs, or 16-bit metadata when m16): part 0 = channels 0-15 (the whole
// slice for g >= 32), part 1 = channels 16-31.
__device__ __forceinline__ void lane_meta(const unsigned char* mrow, int slice, int gshift,
                                          bool m16, float& s0, float& z0, float& s1,
                                          float& z1) {
  if (m16) {
    const uint16_t* mr = reinterpret_cast<const uint16_t*>(mrow);
    uint32_t h0, h1;
    if (gshift >= 5) {
      h0 = h1 = mr[(slice * 32) >> gshift];
    } else {
      h0 = mr[slice * 2];
      h1 = mr[slice * 2 + 1];
    }
    s0 = m16_scale_value(h0 & 0xFFu);
    z0 = m16_offset(h0, s0);
    s1 = m16_scale_value(h1 & 0xFFu);
    z1 = m16_offset(h1, s1);
    return;
  }
  const uint32_t* mr = reinterpret_cast<const uint32_t*>(mrow);
  if (gshift >= 5) {
    unpack_meta(mr[(slice * 32) >> gshift], s0, z0);
    s1 = s0;
    z1 = z0;
  } else {
    const uint2 mw = *reinterpret_cast<const uint2*>(mr + slice * 2);
    unpack_meta(mw.x, s0, z0);
    unpack_meta(mw.y, s1, z1);
  }
}

// q'.D(c) over this lane's 32 channels of one token of one component:
// s~ * sum q'_i c_i + z~ * sum q'_i per group part.
template <int BITS>
__device__ __forceinline__ float comp_dot(const uint32_t* cw, const unsigned char* mrow,
                                          bool m16, int slice, int gshift,
                                          const float (&q)[32], float qsa, float qsb) {
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
    const uint32_t c = (w[slice_word<BITS>(ch)] >> slice_shift<BITS>(ch)) & QMAX;
    if (ch < 16)
      a0 = fmaf(q[ch], code_to_float(c), a0);
    else
      a1 = fmaf(q[ch], code_to_float(c), a1);
  }
  float s0, z0, s1, z1;
  lane_meta(mrow, slice, gshift, m16, s0, z0, s1, z1);
  if (gshift >= 5) return s0 * (a0 + a1) + z0 * (qsa + qsb);
  return s0 * a0 + z0 * qsa + (s1 * a1 + z1 * qsb);
}

// acc += pk * D(c) over this lane's 32 channels; the offsets go to cst0/cst1.
template <int BITS>
__device__ __forceinline__ void comp_acc(const uint32_t* cw, const unsigned char* mrow,
                                         bool m16, int slice, int gshift, float pk,
                                         float (&acc)[32], float& cst0, float& cst1) {
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
  lane_meta(mrow, slice, gshift, m16, s0, z0, s1, z1);
  const float w0 = pk * s0, w1 = pk * s1;
  cst0 = fmaf(pk, z0, cst0);
  cst1 = fmaf(pk, z1, cst1);
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) {
    const uint32_t c = (w[slice_word<BITS>(ch)] >> slice_shift<BITS>(ch)) & QMAX;
    acc[ch] = fmaf(ch < 16 ? w0 : w1, code_to_float(c), acc[ch]);
  }
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
  __shared__ float s_qmu[RQ_MAX_LOOPS][D / 32];   // q'.mu_c per slice (fixed means)

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

  // One copy of kRecsPerStage consecutive records per component and side
  // (stages start at multiples of kChunk tokens, so they never leave the row).
  auto issue = [&](int i) {
    const int s = i % S;
    const int t0 = t_begin + i * kChunk;
    unsigned char* st = smem + static_cast<size_t>(s) * p.stage_bytes;
    uint32_t bytes = 0;
    for (int side = 0; side < 2; ++side) {
      const Comp* cs = side == 0 ? p.k : p.v;
      for (int c = 0; c < p.ncomp; ++c) bytes += kRecsPerStage * cs[c].rec_bytes;
    }
    mbar_arrive_expect_tx(&full_bar[s], bytes);
    for (int side = 0; side < 2; ++side) {
      const Comp* cs = side == 0 ? p.k : p.v;
      for (int c = 0; c < p.ncomp; ++c)
        bulk_copy_g2s(st + map.comp[side][c], comp_record(cs[c], bhi, p.nblk, t0),
                      kRecsPerStage * cs[c].rec_bytes, &full_bar[s]);
    }
  };
  int issued = 0;
  if (t == 0) {
    for (; issued < min(S, nchunks); ++issued) issue(issued);
  }
  const float qrs = rotate_query<D>(
      svec, p.urot_k ? p.urot_k + static_cast<size_t>(bhi % p.heads) * D * D : nullptr,
      p.rot_scale);
  float q[32];
  float qsa = 0.0f, qsb = 0.0f;
  {
    const float sc = qrs * p.scale_log2;
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) {
      q[ch] = svec[slice * 32 + ch] * sc;
      if (ch < 16) qsa += q[ch]; else qsb += q[ch];
    }
  }

  // Fixed means [RQ App. G.2]: q'.mu_c over each 32-channel slice.
  const int head = bhi % p.heads;
  {
    const float sc = qrs * p.scale_log2;
    for (int e = t; e < p.ncomp * G::P; e += kDecodeThreads) {
      const int c = e / G::P, s = e % G::P;
      float sum = 0.0f;
      if (p.k[c].mean != nullptr) {
        const float* mu = p.k[c].mean + static_cast<size_t>(head) * D + s * 32;
        for (int ch = 0; ch < 32; ++ch) sum = fmaf(svec[s * 32 + ch] * sc, mu[ch], sum);
      }
      s_qmu[c][s] = sum;
    }
  }
  __syncthreads();

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
        const int bits = p.k[c].bits, jl = j % kBlock;
        const unsigned char* rec = stage_rec(st, map, p.k[c], 0, c, j);
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(rec) + jl * (D * bits / 32) +
                             slice * bits;
        const bool m16 = p.k[c].meta16 != 0;
        const unsigned char* mr = rec + map.meta[0][c] + jl * (D / p.k[c].group) * (m16 ? 2 : 4);
        const float d = (bits == 4)
                            ? comp_dot<4>(cw, mr, m16, slice, log2_pow2(p.k[c].group), q, qsa, qsb)
                            : comp_dot<2>(cw, mr, m16, slice, log2_pow2(p.k[c].group), q, qsa, qsb);
        part = fmaf(kappa, d, part);
        if (p.k[c].mean != nullptr) part = fmaf(kappa, s_qmu[c][slice], part);
        if (c + 1 < p.ncomp)
          kappa *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(rec + map.alpha[0][c])[jl]);
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
        const int bits = p.v[c].bits, jl = j % kBlock;
        const unsigned char* rec = stage_rec(st, map, p.v[c], 1, c, j);
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(rec) + jl * (D * bits / 32) +
                             slice * bits;
        const bool m16 = p.v[c].meta16 != 0;
        const unsigned char* mr = rec + map.meta[1][c] + jl * (D / p.v[c].group) * (m16 ? 2 : 4);
        if (bits == 4)
          comp_acc<4>(cw, mr, m16, slice, log2_pow2(p.v[c].group), kappa, acc, cst0, cst1);
        else
          comp_acc<2>(cw, mr, m16, slice, log2_pow2(p.v[c].group), kappa, acc, cst0, cst1);
        if (p.v[c].mean != nullptr) {
          const float* mu = p.v[c].mean + static_cast<size_t>(head) * D + slice * 32;
#pragma unroll
          for (int ch = 0; ch < 32; ++ch) acc[ch] = fmaf(kappa, __ldg(mu + ch), acc[ch]);
        }
        if (c + 1 < p.ncomp)
          kappa *= bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(rec + map.alpha[1][c])[jl]);
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
  const bool aborted = __syncthreads_or(s_abort != 0) != 0;
  finish_split<D, kDecodeThreads, Geom<D>::NSLOT, true>(
      m, l, acc, slice, slot, reinterpret_cast<float*>(smem), bhi, split, p.splits, p.partials,
      p.counters, p.q, p.kcur, p.vcur, p.scale_log2, p.rot_scale, p.out, svec, sred, aborted,
      p.urot_v ? p.urot_v + static_cast<size_t>(bhi % p.heads) * D * D : nullptr);
}

template <int D>
size_t scratch_bytes() {
  return (Geom<D>::NSLOT * red_pitch<D>() + 2 * Geom<D>::NSLOT) * sizeof(float);
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
  size_t scr = D == 64 ? scratch_bytes<64>() : scratch_bytes<128>();
  if (scr < 3 * 1024 * sizeof(float)) scr = 3 * 1024 * sizeof(float);   // split headers
  return ring > scr ? ring : scr;
}

cudaError_t decode_occupancy(int D, size_t dyn_smem, int* ctas_per_sm) {
  cudaError_t e;
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

}  // namespace rq
