// rq_quantize.cu -- quantise-and-append kernels (anchor and LS residual) and
// the reconstruction kernel used for export / tests.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// Thread mapping: a row (one token of one head, D channels) is owned by
// P = D/32 consecutive lanes; lane `slice` of the row holds channels
// [32*slice, 32*slice + 32) in registers.  The Hadamard transform runs its
// first five butterfly stages inside the lane and the remaining log2(P)
// stages across lanes with xor-shuffles; group min/max and the two dot
// products of the LS coefficient are lane-serial followed by xor-shuffle
// butterflies.  Every floating-point step that decides a stored bit uses an
// explicitly rounded intrinsic (no contraction), in this fixed order:
//   Hadamard stages h = 1, 2, ..., D/2 with (a + b, a - b), then one multiply
//   by fp32(1/sqrt(D)); dots: per-lane serial fma from +0, then butterflies
//   with xor offsets P/2, ..., 1; alpha = dot(z, R) / dot(R, R);
//   E = fma(-bf16(alpha), R, z); group: mn, mx (+0 for zeros),
//   s = (mx - mn) / (2^b - 1), s~ = fp16(s), z~ = fp16(mn), inv = 1/s~,
//   code = rint_even(clamp((x - z~) * inv, 0, 2^b - 1)).
#include "rq_internal.cuh"

namespace rq {
namespace {

constexpr int kQuantThreads = 256;

// Normalised-free Sylvester-Hadamard butterflies over one row held as
// P x 32 registers (lane `slice` holds channels 32*slice .. 32*slice+31).
template <int D>
__device__ __forceinline__ void fwht_row(float (&z)[32], int slice) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = z[j], b = z[j + h];
        z[j] = __fadd_rn(a, b);
        z[j + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int hl = 1; hl < D / 32; hl <<= 1) {
    const bool upper = (slice & hl) != 0;   // this lane holds the "a - b" half
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, z[k], hl);
      z[k] = upper ? __fsub_rn(o, z[k]) : __fadd_rn(z[k], o);
    }
  }
}

// Stored levels fma(s~, code, z~) of one lane's 32 channels of a component
// at token t of row `row`.
template <int BITS>
__device__ __forceinline__ void deq_slice_t(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                            int slice, int D, float (&o)[32]) {
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  unsigned char* rec = comp_record(c, row, nblk, t);
  const int i = static_cast<int>(t % kBlock);
  const uint32_t* w = rec_codes(rec, D, BITS, i) + slice * BITS;
  uint32_t words[BITS];
#pragma unroll
  for (int k = 0; k < BITS; ++k) words[k] = w[k];
  const uint32_t* m = rec_meta(rec, D, BITS, c.group, i);
  uint32_t mw0, mw1;
  if (c.group >= 32) {
    mw0 = m[(slice * 32) / c.group];
    mw1 = mw0;
  } else {  // group 16: two groups per lane
    mw0 = m[slice * 2];
    mw1 = m[slice * 2 + 1];
  }
  const float s0 = __half2float(__ushort_as_half((unsigned short)(mw0 & 0xFFFFu)));
  const float z0 = __half2float(__ushort_as_half((unsigned short)(mw0 >> 16)));
  const float s1 = __half2float(__ushort_as_half((unsigned short)(mw1 & 0xFFFFu)));
  const float z1 = __half2float(__ushort_as_half((unsigned short)(mw1 >> 16)));
#pragma unroll
  for (int ch = 0; ch < 32; ++ch) {
    const uint32_t code = (words[slice_word<BITS>(ch)] >> slice_shift<BITS>(ch)) & QMAX;
    const float cf = static_cast<float>(code);
    o[ch] = (ch < 16) ? __fmaf_rn(s0, cf, z0) : __fmaf_rn(s1, cf, z1);
  }
}

__device__ __forceinline__ void deq_slice(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                          int slice, int D, float (&o)[32]) {
  if (c.bits == 4)
    deq_slice_t<4>(c, row, nblk, t, slice, D, o);
  else
    deq_slice_t<2>(c, row, nblk, t, slice, D, o);
}

// Rotated reconstruction of a chain [0 .. n-1] (anchor last) at token t of
// row `row`: Z = deq(anchor); for k = n-2 .. 0: Z = fma(alpha~_k, Z, deq_k).
__device__ __forceinline__ void chain_slice(const Comp* comps, int n, int64_t row, int64_t nblk,
                                            int64_t t, int slice, int D, float (&zr)[32]) {
  deq_slice(comps[n - 1], row, nblk, t, slice, D, zr);
  for (int k = n - 2; k >= 0; --k) {
    float d[32];
    deq_slice(comps[k], row, nblk, t, slice, D, d);
    const Comp& c = comps[k];
    const float a = bf16_bits_to_f32(
        *rec_alpha(comp_record(c, row, nblk, t), D, c.bits, c.group, static_cast<int>(t % kBlock)));
#pragma unroll
    for (int ch = 0; ch < 32; ++ch) zr[ch] = __fmaf_rn(a, zr[ch], d[ch]);
  }
}

// Affine quantisation [RQ §2.1] of one lane's 32 values and the packed store;
// if `levels` is given it receives the stored levels fma(s~, code, z~) (what
// a reader of the record reconstructs).
template <int D, int BITS, int G>
__device__ __forceinline__ void quantize_store(const float (&z)[32], int slice,
                                               bool active, uint32_t* codes_row,
                                               uint32_t* meta_row, float* levels = nullptr) {
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  constexpr int GL = G < 32 ? G : 32;    // group part held by this lane
  constexpr int NG = 32 / GL;            // group parts per lane
  constexpr int LPG = G > 32 ? G / 32 : 1;  // lanes sharing a group
  uint32_t words[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) words[i] = 0u;
  uint32_t metaw[NG];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    float mn = z[gi * GL], mx = z[gi * GL];
#pragma unroll
    for (int k = 1; k < GL; ++k) {
      mn = fminf(mn, z[gi * GL + k]);
      mx = fmaxf(mx, z[gi * GL + k]);
    }
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    mn = __fadd_rn(mn, 0.0f);   // a zero end of the range is +0
    mx = __fadd_rn(mx, 0.0f);
    const float s = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(QMAX));
    const __half sh = __float2half_rn(s);
    const __half zh = __float2half_rn(mn);
    const float st = __half2float(sh);
    const float zt = __half2float(zh);
    const float inv = (st > 0.0f) ? __fdiv_rn(1.0f, st) : 0.0f;
    metaw[gi] = static_cast<uint32_t>(__half_as_ushort(sh)) |
                (static_cast<uint32_t>(__half_as_ushort(zh)) << 16);
#pragma unroll
    for (int k = 0; k < GL; ++k) {
      const int ch = gi * GL + k;
      float u = __fmul_rn(__fsub_rn(z[ch], zt), inv);
      u = fminf(fmaxf(u, 0.0f), static_cast<float>(QMAX));
      // u + 1.5*2^23 rounds u to the nearest integer, ties to even, and
      // leaves that integer in the low mantissa bits.
      const uint32_t code = __float_as_uint(__fadd_rn(u, 12582912.0f)) & QMAX;
      words[slice_word<BITS>(ch)] |= code << slice_shift<BITS>(ch);
      if (levels != nullptr) levels[ch] = __fmaf_rn(st, static_cast<float>(code), zt);
    }
  }
  if (!active) return;
  uint32_t* cw = codes_row + slice * BITS;
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(cw) = make_uint4(words[0], words[1], words[2], words[3]);
  } else {
    *reinterpret_cast<uint2*>(cw) = make_uint2(words[0], words[1]);
  }
  if constexpr (NG == 2) {
    *reinterpret_cast<uint2*>(meta_row + slice * 2) = make_uint2(metaw[0], metaw[1]);
  } else if constexpr (LPG == 1) {
    meta_row[slice] = metaw[0];
  } else {
    if ((slice % LPG) == 0) meta_row[slice / LPG] = metaw[0];
  }
}

// Row of bf16 x -> fp32 -> Z = H x (normalised) in one lane's 32 registers.
template <int D>
__device__ __forceinline__ void load_rotate(const uint16_t* xrow, bool active, int slice,
                                            float rot_scale, float (&z)[32]) {
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(xrow + slice * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = src[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        z[i * 8 + 2 * j] = __uint_as_float(w[j] << 16);
        z[i * 8 + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) z[k] = 0.0f;
  }
  fwht_row<D>(z, slice);
#pragma unroll
  for (int k = 0; k < 32; ++k) z[k] = __fmul_rn(z[k], rot_scale);
}

// Least-squares coefficient of z against the reference over the row
// [RQ §3.2 scaling coefficient, App. G.1]: alpha~ = bf16(<z, ref> / <ref, ref>)
// (0 for a zero reference); z becomes the residual fma(-alpha~, ref, z).
template <int D>
__device__ __forceinline__ __nv_bfloat16 ls_residual(float (&z)[32], const float (&ref)[32]) {
  constexpr int P = D / 32;
  float dzr = 0.0f, drr = 0.0f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    dzr = __fmaf_rn(z[k], ref[k], dzr);
    drr = __fmaf_rn(ref[k], ref[k], drr);
  }
#pragma unroll
  for (int off = P / 2; off >= 1; off >>= 1) {
    dzr = __fadd_rn(dzr, __shfl_xor_sync(0xffffffffu, dzr, off));
    drr = __fadd_rn(drr, __shfl_xor_sync(0xffffffffu, drr, off));
  }
  const float a = (drr > 0.0f) ? __fdiv_rn(dzr, drr) : 0.0f;
  const __nv_bfloat16 ab = __float2bfloat16_rn(a);
  const float at = __bfloat162float(ab);
#pragma unroll
  for (int k = 0; k < 32; ++k) z[k] = __fmaf_rn(-at, ref[k], z[k]);
  return ab;
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_kernel(const __grid_constant__ QuantParams p) {
  constexpr int P = D / 32;
  constexpr int RPW = 32 / P;
  const int lane = threadIdx.x & 31;
  const int slice = lane % P;
  const int64_t total = static_cast<int64_t>(p.bh) * p.n;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) +
                       (threadIdx.x >> 5);
  for (int64_t base = warp * RPW; base < total; base += nwarps * RPW) {
    const int64_t row = base + lane / P;
    const bool active = row < total;
    float z[32];
    load_rotate<D>(p.x + (active ? row : 0) * D, active, slice, p.rot_scale, z);

    const int64_t bhi = active ? row / p.n : 0;
    const int64_t t = p.t0 + (active ? row % p.n : 0);

    if (p.dst.has_alpha) {
      // Least-squares coefficient against the reconstructed reference
      // [RQ §3.2 scaling coefficient, App. G.1], then the residual.
      float ref[32];
      if (active) {
        chain_slice(p.ref, p.nref, bhi, p.nblk, t, slice, D, ref);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ref[k] = 0.0f;
      }
      const __nv_bfloat16 ab = ls_residual<D>(z, ref);
      if (active && slice == 0)
        *rec_alpha(comp_record(p.dst, bhi, p.nblk, t), D, BITS, G, static_cast<int>(t % kBlock)) =
            __bfloat16_as_ushort(ab);
    }
    unsigned char* rec = comp_record(p.dst, bhi, p.nblk, t);
    const int i = static_cast<int>(t % kBlock);
    quantize_store<D, BITS, G>(z, slice, active, rec_codes(rec, D, BITS, i),
                               rec_meta(rec, D, BITS, G, i));
  }
}

// Quantisation of one component at token t (run-time bits / group): codes,
// metadata and (if `levels`) the stored levels of this lane's 32 channels.
template <int D>
__device__ __forceinline__ void quantize_comp(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                              const float (&z)[32], int slice, bool active,
                                              float* levels) {
  unsigned char* rec = comp_record(c, row, nblk, t);
  const int i = static_cast<int>(t % kBlock);
  uint32_t* cw = rec_codes(rec, D, c.bits, i);
  uint32_t* mw = rec_meta(rec, D, c.bits, c.group, i);
  const int key = c.bits * 1000 + c.group;
  switch (key) {
    case 2016: quantize_store<D, 2, 16>(z, slice, active, cw, mw, levels); break;
    case 2032: quantize_store<D, 2, 32>(z, slice, active, cw, mw, levels); break;
    case 2064: quantize_store<D, 2, 64>(z, slice, active, cw, mw, levels); break;
    case 4016: quantize_store<D, 4, 16>(z, slice, active, cw, mw, levels); break;
    case 4032: quantize_store<D, 4, 32>(z, slice, active, cw, mw, levels); break;
    case 4064: quantize_store<D, 4, 64>(z, slice, active, cw, mw, levels); break;
    default:
      if constexpr (D >= 128) {
        if (key == 2128) quantize_store<D, 2, 128>(z, slice, active, cw, mw, levels);
        else if (key == 4128) quantize_store<D, 4, 128>(z, slice, active, cw, mw, levels);
      }
      break;
  }
}

// Every loop of a (layer, token range) for one side (blockIdx.y): the anchor
// is quantised first and its stored levels stay in registers as the
// reference; each residual loop then takes its LS coefficient, residual and
// quantisation against it [RQ §3.2, §3.4, App. G.1].  Under the Next-loop
// policy the loops run from L-2 down to 0 and the reference becomes
// Z^_r = fma(alpha~_r, Z^_{r+1}, D(c_r)) after loop r.  The anchor is read
// once and never re-read from the cache; the arithmetic (and so every
// stored bit) is that of the per-loop kernels.
template <int D>
__global__ void __launch_bounds__(kQuantThreads, 2)
    quantize_loops_kernel(const __grid_constant__ QuantLoopsParams p) {
  constexpr int P = D / 32;
  constexpr int RPW = 32 / P;
  const int side = blockIdx.y;
  const uint16_t* xs = p.x[side];
  if (xs == nullptr) return;
  const int lane = threadIdx.x & 31;
  const int slice = lane % P;
  const int64_t total = static_cast<int64_t>(p.bh) * p.n;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) +
                       (threadIdx.x >> 5);
  const int a = p.nloops - 1;
  for (int64_t base = warp * RPW; base < total; base += nwarps * RPW) {
    const int64_t row = base + lane / P;
    const bool active = row < total;
    const int64_t r_in = active ? row : 0;
    const int64_t bhi = active ? row / p.n : 0;
    const int64_t t = p.t0 + (active ? row % p.n : 0);
    float ref[32], z[32];
    load_rotate<D>(xs + (static_cast<int64_t>(a) * total + r_in) * D, active, slice, p.rot_scale,
                   z);
    quantize_comp<D>(p.dst[side][a], bhi, p.nblk, t, z, slice, active, ref);
    for (int k = 0; k < a; ++k) {
      const int r = p.chained ? a - 1 - k : k;
      const Comp& c = p.dst[side][r];
      load_rotate<D>(xs + (static_cast<int64_t>(r) * total + r_in) * D, active, slice,
                     p.rot_scale, z);
      const __nv_bfloat16 ab = ls_residual<D>(z, ref);
      if (active && slice == 0)
        *rec_alpha(comp_record(c, bhi, p.nblk, t), D, c.bits, c.group,
                   static_cast<int>(t % kBlock)) = __bfloat16_as_ushort(ab);
      float lv[32];
      quantize_comp<D>(c, bhi, p.nblk, t, z, slice, active, lv);
      if (p.chained) {
        const float at = __bfloat162float(ab);
#pragma unroll
        for (int ch = 0; ch < 32; ++ch) ref[ch] = __fmaf_rn(at, ref[ch], lv[ch]);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
    dequantize_kernel(const __grid_constant__ DequantParams p) {
  constexpr int P = D / 32;
  constexpr int RPW = 32 / P;
  const int lane = threadIdx.x & 31;
  const int slice = lane % P;
  const int64_t total = static_cast<int64_t>(p.bh) * p.n;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) +
                       (threadIdx.x >> 5);
  for (int64_t base = warp * RPW; base < total; base += nwarps * RPW) {
    const int64_t row = base + lane / P;
    const bool active = row < total;
    float z[32];
    if (active) {
      chain_slice(p.comp, p.ncomp, row / p.n, p.nblk, p.t0 + row % p.n, slice, D, z);
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) z[k] = 0.0f;
    }
    // X^ = H^T Z^ = H Z^ (the normalised Sylvester matrix is symmetric).
    fwht_row<D>(z, slice);
    if (active) {
      float4* dst = reinterpret_cast<float4*>(p.out + row * D + slice * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(z[4 * i] * p.rot_scale, z[4 * i + 1] * p.rot_scale,
                             z[4 * i + 2] * p.rot_scale, z[4 * i + 3] * p.rot_scale);
    }
  }
}

int quant_grid(int64_t rows, int D) {
  const int rows_per_cta = (kQuantThreads / 32) * (32 / (D / 32));
  int64_t ctas = (rows + rows_per_cta - 1) / rows_per_cta;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = static_cast<int64_t>(sms) * 8;   // resident CTAs at 256 threads
  if (ctas > cap) ctas = cap;
  return static_cast<int>(ctas < 1 ? 1 : ctas);
}

template <int D, int BITS, int G>
cudaError_t launch_q(const QuantParams& p, cudaStream_t s) {
  const int grid = quant_grid(static_cast<int64_t>(p.bh) * p.n, D);
  quantize_kernel<D, BITS, G><<<grid, kQuantThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_q_group(const QuantParams& p, int group, cudaStream_t s) {
  switch (group) {
    case 16: return launch_q<D, BITS, 16>(p, s);
    case 32: return launch_q<D, BITS, 32>(p, s);
    case 64: return launch_q<D, BITS, 64>(p, s);
    case 128: if constexpr (D >= 128) return launch_q<D, BITS, 128>(p, s); else return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t launch_q_bits(const QuantParams& p, int bits, int group, cudaStream_t s) {
  if (bits == 2) return launch_q_group<D, 2>(p, group, s);
  if (bits == 4) return launch_q_group<D, 4>(p, group, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quantize(const QuantParams& p, int D, int bits, int group,
                            cudaStream_t s) {
  if (static_cast<int64_t>(p.bh) * p.n == 0) return cudaSuccess;
  if (D == 64) return launch_q_bits<64>(p, bits, group, s);
  if (D == 128) return launch_q_bits<128>(p, bits, group, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_loops(const QuantLoopsParams& p, int D, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.bh) * p.n;
  if (rows == 0) return cudaSuccess;
  const dim3 grid(quant_grid(rows, D), 2);
  if (D == 64)
    quantize_loops_kernel<64><<<grid, kQuantThreads, 0, s>>>(p);
  else if (D == 128)
    quantize_loops_kernel<128><<<grid, kQuantThreads, 0, s>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const DequantParams& p, int D, cudaStream_t s) {
  if (static_cast<int64_t>(p.bh) * p.n == 0) return cudaSuccess;
  const int grid = quant_grid(static_cast<int64_t>(p.bh) * p.n, D);
  if (D == 64)
    dequantize_kernel<64><<<grid, kQuantThreads, 0, s>>>(p);
  else if (D == 128)
    dequantize_kernel<128><<<grid, kQuantThreads, 0, s>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace rq
