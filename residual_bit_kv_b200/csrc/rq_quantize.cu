// rq_quantize.cu -- quantise-and-append kernels (anchor and LS residual) and
// the reconstruction kernel used for export / tests.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
//
// Thread mapping: a row (one token of one head, D channels) is owned by
// P = D/32 consecutive lanes; lane `slice` of the row holds channels
// [32*slice, 32*slice + 32) in registers as 16 packed fp32 pairs
// v[k] = (channel k, channel k + 16) of the slice, so that the butterflies,
// the scaling, the residual and the quantisation run as packed fp32
// operations (each element of a pair rounded exactly as its scalar op).  The Hadamard transform runs its
// first five butterfly stages inside the lane and the remaining log2(P)
// stages across lanes with xor-shuffles; the group min/max are trees of
// three-input min/max (exact in any order) and the two dot products of the
// LS coefficient are lane-serial followed by xor-shuffle butterflies.  The
// fused all-loops kernel streams its input rows through a per-warp
// shared-memory ring filled by cp.async ahead of use; the per-loop kernel
// rebuilds a residual's reference before loading the row, which keeps it at
// two CTAs of 256 threads per SM.  Every floating-point step that decides a stored bit uses an
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
constexpr float kRoundMagic = 12582912.0f;       // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Channel k of a slice held as pairs v[k mod 16].(x if k < 16 else y).
__device__ __forceinline__ float ch_of(const float2 (&v)[16], int k) {
  return k < 16 ? v[k].x : v[k - 16].y;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);   // RN(a - b)
}

// Normalisation-free Sylvester-Hadamard butterflies over one row (stages
// h = 1, 2, ..., D/2 in order): h = 1..8 pair-wise on v, h = 16 inside each
// pair, h >= 32 across lanes by xor shuffles.
template <int D>
__device__ __forceinline__ void fwht_row(float2 (&v)[16], int slice) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & h) continue;
      const float2 a = v[i], b = v[i + h];
      v[i] = __fadd2_rn(a, b);
      v[i + h] = sub2(a, b);
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float a = v[k].x, b = v[k].y;
    v[k] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int hl = 1; hl < D / 32; hl <<= 1) {
    // this lane holds the "a - b" half when (slice & hl): RN(s * mine + other)
    const float sg = (slice & hl) ? -1.0f : 1.0f;
    const float2 s2 = make_float2(sg, sg);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[k].x, hl),
                                   __shfl_xor_sync(0xffffffffu, v[k].y, hl));
      v[k] = __ffma2_rn(v[k], s2, o);
    }
  }
}

// One lane's 32 bf16 channels (four 16-byte pieces, channels 8i .. 8i + 7 in
// piece i) -> fp32 pairs -> Z = H x (normalised) in the lane's 16 pairs.
template <int D>
__device__ __forceinline__ void rotate_pieces(const uint4 (&q)[4], bool active, int slice,
                                              float rot_scale, float2 (&v)[16]) {
  if (active) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c0 = i * 8 + 2 * j;   // channels c0, c0 + 1
        const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
        if (c0 < 16) {
          v[c0].x = lo;
          v[c0 + 1].x = hi;
        } else {
          v[c0 - 16].y = lo;
          v[c0 - 15].y = hi;
        }
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = make_float2(0.0f, 0.0f);
  }
  fwht_row<D>(v, slice);
  const float2 rs = make_float2(rot_scale, rot_scale);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __fmul2_rn(v[k], rs);
}

// Row of bf16 x (global memory) -> Z = H x in one lane's 16 pairs.
template <int D>
__device__ __forceinline__ void load_rotate(const uint16_t* xrow, bool active, int slice,
                                            float rot_scale, float2 (&v)[16]) {
  uint4 q[4];
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(xrow + slice * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = src[i];
  }
  rotate_pieces<D>(q, active, slice, rot_scale, v);
}

// Dense rotation [RQ §3.3, App. G.1, App. G.2]: Z = U x for the warp's eight
// rows (head_dim 128; the row of lane l is l / 4, its slice l % 4), U the
// binary16 matrix of the row's head (row i = output channel i), x rounded
// from bf16 to binary16, fp32 accumulation on the tensor cores
// (mma.m16n8k16, rows 8..15 of A unused).  Both contraction indices are
// permuted so that no data moves between lanes:
//   k: step ks, A/B fragment column 2t + e (+8) <-> channel 32t + 4ks + e (+2),
//      so a lane's A fragments are its own slice, words 2ks and 2ks + 1;
//   n: tile nt, column c <-> output channel 32 (c >> 1) + 2 nt + (c & 1),
//      so the accumulators of lane (g, t) are channels 32t + 2nt + {0, 1} of
//      its own row, and its B fragments are 64 contiguous bytes of U row
//      32 (g >> 1) + 2 nt + (g & 1).
// A warp whose rows belong to several heads runs one pass per head; a lane
// keeps the pass of its own head (rows are independent in the product).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Per-lane staging of the dense rotation's accumulators (a stride of 34
// floats keeps the float2 stores of a warp on distinct bank pairs).
constexpr int kDenseLaneFloats = 34;
constexpr int kDenseTileBytes = (kQuantThreads) * kDenseLaneFloats * 4;

// A CTA's copy of one head's matrix in shared memory: rows of 128 binary16
// padded to 136 (272 bytes), so the four 16-byte loads of a quarter-warp
// (two U rows, four lanes) fall in at most two wavefronts.
constexpr int kUshStride = 136;
constexpr int kUshBytes = 128 * kUshStride * 2;

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
  return r;
}

template <int D>
__device__ __forceinline__ void rotate_dense(const uint4 (&q)[4], bool active, int lane, int head,
                                             const uint16_t* urot, float* tile,
                                             float2 (&v)[16], uint32_t ush = 0u,
                                             int ush_head = -1) {
  static_assert(D == 128, "the dense rotation is built for head_dim 128");
  const int g = lane >> 2, t = lane & 3;
  uint32_t a[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) a[4 * i + j] = active ? bf16x2_to_f16x2(w[j]) : 0u;
  }
  uint32_t todo = __ballot_sync(0xffffffffu, active);
  while (todo != 0u) {
    const int h = __shfl_sync(0xffffffffu, head, __ffs(todo) - 1);
    const bool mine = active && head == h;
    todo &= ~__ballot_sync(0xffffffffu, mine);
    if (h == ush_head) {
      // the CTA's shared copy of this head's matrix
      const uint32_t ub = ush + ((32 * (g >> 1) + (g & 1)) * kUshStride + 32 * t) * 2;
#pragma unroll 2
      for (int nt = 0; nt < 16; ++nt) {
        const uint32_t un = ub + nt * 2 * kUshStride * 2;
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 bw = lds128(un + 16 * i);
          mma_16816(d, a[4 * i], a[4 * i + 1], bw.x, bw.y);
          mma_16816(d, a[4 * i + 2], a[4 * i + 3], bw.z, bw.w);
        }
        if (mine) *reinterpret_cast<float2*>(tile + 2 * nt) = make_float2(d[0], d[1]);
      }
      continue;
    }
    // U row of n-tile nt for this lane: 64 bytes; the next tile's row is
    // loaded while the current one's products run
    const uint4* up = reinterpret_cast<const uint4*>(
        urot + static_cast<size_t>(h) * D * D + 32 * t +
        static_cast<size_t>(32 * (g >> 1) + (g & 1)) * D);
    uint4 bn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) bn[i] = __ldg(up + i);
#pragma unroll 1
    for (int nt = 0; nt < 16; ++nt) {
      uint4 bc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) bc[i] = bn[i];
      if (nt + 1 < 16) {
        const uint4* un = up + (nt + 1) * (2 * D / 8);   // two U rows further per tile
#pragma unroll
        for (int i = 0; i < 4; ++i) bn[i] = __ldg(un + i);
      }
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {   // 16 bytes of U serve two k-steps
        mma_16816(d, a[4 * i], a[4 * i + 1], bc[i].x, bc[i].y);
        mma_16816(d, a[4 * i + 2], a[4 * i + 3], bc[i].z, bc[i].w);
      }
      if (mine) *reinterpret_cast<float2*>(tile + 2 * nt) = make_float2(d[0], d[1]);
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k)
    v[k] = active ? make_float2(tile[k], tile[k + 16]) : make_float2(0.0f, 0.0f);
}

// Input staging of the fused kernel: each warp streams its rows through a
// private ring of kQStages shared-memory slots of 32 x 64 bytes (the RPW
// rows of one loop: 8 rows of 128 channels or 16 rows of 64), filled by
// 16-byte cp.async copies kQStages - 1 jobs ahead of the job being
// quantised, so every warp keeps about 6 KB of input in flight without
// holding it in registers (the dense-rotation instantiation keeps two slots,
// to leave room for its shared matrix).  A copy instruction covers 512 contiguous bytes
// (lane l: bytes 16 l of each 512-byte quarter); piece pi of the slice
// that lane l of the row reads lands at pi ^ ((l >> 1) & 3), so the four
// 16-byte reads of a quarter-warp hit eight distinct bank groups.
constexpr int kQStages = 4;
constexpr int kQSlotBytes = 2048;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copies `rows` (<= RPW) consecutive rows of D bf16 from src into a slot.
template <int D>
__device__ __forceinline__ void stage_rows(uint32_t slot, const unsigned char* src, int rows,
                                           int lane) {
  constexpr int P = D / 32;
  const int nbytes = rows * D * 2;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = i * 512 + lane * 16;
    if (o < nbytes) {
      const int rho = o / (2 * D), b = o % (2 * D);
      const int sg = b / 64, pi = (b % 64) / 16;
      const int l = rho * P + sg;
      cp_async16(slot + rho * 2 * D + sg * 64 + ((pi ^ ((l >> 1) & 3)) << 4), src + o);
    }
  }
}

// This lane's four pieces of its row from a filled slot.
template <int D>
__device__ __forceinline__ void read_slot(uint32_t slot, int lane, uint4 (&q)[4]) {
  constexpr int P = D / 32;
  const uint32_t a = slot + (lane / P) * 2 * D + (lane % P) * 64;
  const int f = (lane >> 1) & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(q[i].x), "=r"(q[i].y), "=r"(q[i].z), "=r"(q[i].w)
                 : "r"(a + ((i ^ f) << 4)));
}

// Stored levels fma(s~, code, z~) of one lane's 32 channels of a component
// at token t of row `row`.
template <int BITS>
__device__ __forceinline__ void deq_slice_t(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                            int slice, int D, float2 (&o)[16]) {
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  unsigned char* rec = comp_record(c, row, nblk, t);
  const int i = static_cast<int>(t % kBlock);
  const uint32_t* w = rec_codes(rec, D, BITS, i) + slice * BITS;
  uint32_t words[BITS];
#pragma unroll
  for (int k = 0; k < BITS; ++k) words[k] = w[k];
  float2 s2, z2;
  if (c.meta16) {
    const uint16_t* m = rec_meta16(rec, D, BITS, c.group, i);
    uint32_t h0, h1;
    if (c.group >= 32) {
      h0 = m[(slice * 32) / c.group];
      h1 = h0;
    } else {  // group 16: two groups per lane
      h0 = m[slice * 2];
      h1 = m[slice * 2 + 1];
    }
    s2 = make_float2(m16_scale_value(h0 & 0xFFu), m16_scale_value(h1 & 0xFFu));
    z2 = make_float2(m16_offset(h0, s2.x), m16_offset(h1, s2.y));
  } else {
    const uint32_t* m = rec_meta(rec, D, BITS, c.group, i);
    uint32_t mw0, mw1;
    if (c.group >= 32) {
      mw0 = m[(slice * 32) / c.group];
      mw1 = mw0;
    } else {  // group 16: two groups per lane
      mw0 = m[slice * 2];
      mw1 = m[slice * 2 + 1];
    }
    s2 = make_float2(__half2float(__ushort_as_half((unsigned short)(mw0 & 0xFFFFu))),
                     __half2float(__ushort_as_half((unsigned short)(mw1 & 0xFFFFu))));
    z2 = make_float2(__half2float(__ushort_as_half((unsigned short)(mw0 >> 16))),
                     __half2float(__ushort_as_half((unsigned short)(mw1 >> 16))));
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t c0 = (words[slice_word<BITS>(k)] >> slice_shift<BITS>(k)) & QMAX;
    const uint32_t c1 = (words[slice_word<BITS>(k + 16)] >> slice_shift<BITS>(k + 16)) & QMAX;
    o[k] = __ffma2_rn(s2, make_float2(static_cast<float>(c0), static_cast<float>(c1)), z2);
  }
}

__device__ __forceinline__ void deq_slice(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                          int slice, int D, float2 (&o)[16]) {
  if (c.bits == 4)
    deq_slice_t<4>(c, row, nblk, t, slice, D, o);
  else
    deq_slice_t<2>(c, row, nblk, t, slice, D, o);
}

// This lane's 32 channels of a component's fixed mean (row `row` uses the
// mean of head row % heads), as pairs (channel k, channel k + 16).
__device__ __forceinline__ void mean_slice(const Comp& c, int64_t row, int slice, int D,
                                           float2 (&m)[16]) {
  const float4* src =
      reinterpret_cast<const float4*>(c.mean + (row % c.heads) * D + slice * 32);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 q = src[i];
    const float e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ch = 4 * i + j;
      if (ch < 16)
        m[ch].x = e[j];
      else
        m[ch - 16].y = e[j];
    }
  }
}

// v <- v - mean (the encoder's mean removal), v <- v + mean (reconstruction).
__device__ __forceinline__ void sub_mean(const Comp& c, int64_t row, int slice, int D,
                                         float2 (&v)[16]) {
  float2 m[16];
  mean_slice(c, row, slice, D, m);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __fadd2_rn(v[k], make_float2(-m[k].x, -m[k].y));
}
__device__ __forceinline__ void add_mean(const Comp& c, int64_t row, int slice, int D,
                                         float2 (&v)[16]) {
  float2 m[16];
  mean_slice(c, row, slice, D, m);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __fadd2_rn(v[k], m[k]);
}

// Rotated reconstruction of a chain [0 .. n-1] (anchor last) at token t of
// row `row`: Z = deq(anchor); for k = n-2 .. 0: Z = fma(alpha~_k, Z, deq_k)
// (+ mu_k when the loop has a fixed mean).
__device__ __forceinline__ void chain_slice(const Comp* comps, int n, int64_t row, int64_t nblk,
                                            int64_t t, int slice, int D, float2 (&zr)[16]) {
  deq_slice(comps[n - 1], row, nblk, t, slice, D, zr);
  for (int k = n - 2; k >= 0; --k) {
    float2 d[16];
    deq_slice(comps[k], row, nblk, t, slice, D, d);
    const Comp& c = comps[k];
    const float a = bf16_bits_to_f32(
        *rec_alpha(comp_record(c, row, nblk, t), D, c.bits, c.group, static_cast<int>(t % kBlock),
                   c.meta16 ? 2 : 4));
    const float2 a2 = make_float2(a, a);
#pragma unroll
    for (int j = 0; j < 16; ++j) zr[j] = __ffma2_rn(a2, zr[j], d[j]);
    if (c.mean != nullptr) add_mean(c, row, slice, D, zr);
  }
}

// Sum over the channels of one packed word of (kRoundMagicBits << shift),
// mod 2^32: what packing the rounded floats' bit patterns adds on top of
// the codes.
template <int BITS>
__host__ __device__ constexpr uint32_t magic_pack_offset(int word) {
  uint32_t o = 0u;
  for (int ch = 0; ch < 32; ++ch)
    if (slice_word<BITS>(ch) == word) o += kRoundMagicBits << slice_shift<BITS>(ch);
  return o;
}

// Codes of one lane's 32 values packed into BITS words: u = (x - z~) * (1/s~)
// clamped to [0, 2^b - 1] (CLAMP 2), or to [0, inf) when the group's ends are
// known to map into [-1/2, 2^b - 1/2) (CLAMP 1: every u then rounds into
// [0, 2^b - 1], so the upper bound changes nothing); u + 1.5 * 2^23 rounds it to the
// nearest integer (ties to even), held in the low mantissa bits of a float
// whose bit pattern is kRoundMagicBits + code; packing adds that pattern
// shifted into place (the magic offsets are subtracted up front), one
// integer multiply-add per code.  LEVELS: `levels` receives fma(s~, code, z~).
template <int BITS, int CLAMP, bool LEVELS>
__device__ __forceinline__ void pack_codes(const float2 (&v)[16], float2 nz, float2 iv,
                                           const float (&st)[2], const float (&zt)[2],
                                           uint32_t (&words)[BITS], float2* levels) {
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  const float2 mg = make_float2(kRoundMagic, kRoundMagic);
  // two partial sums per word (even and odd k) keep the add chains short;
  // the fields never overlap, so any grouping of the adds gives the same word
  uint32_t odd[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) {
    words[i] = 0u - magic_pack_offset<BITS>(i);
    odd[i] = 0u;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    uint32_t* wk = (k & 1) ? odd : words;
    float2 u = __fmul2_rn(__fadd2_rn(v[k], nz), iv);
    if constexpr (CLAMP == 2) {
      u.x = fminf(fmaxf(u.x, 0.0f), static_cast<float>(QMAX));
      u.y = fminf(fmaxf(u.y, 0.0f), static_cast<float>(QMAX));
    } else {
      // the group's ends already map into [-1/2, 2^b - 1/2): only the
      // lower bound is applied (it changes no code there), which also keeps
      // the rounding add a separate operation from the multiply
      u.x = fmaxf(u.x, 0.0f);
      u.y = fmaxf(u.y, 0.0f);
    }
    const float2 r = __fadd2_rn(u, mg);
    const uint32_t b0 = __float_as_uint(r.x), b1 = __float_as_uint(r.y);
    wk[slice_word<BITS>(k)] += b0 << slice_shift<BITS>(k);
    wk[slice_word<BITS>(k + 16)] += b1 << slice_shift<BITS>(k + 16);
    if constexpr (LEVELS) {
      const float2 cf = __fadd2_rn(r, make_float2(-kRoundMagic, -kRoundMagic));   // exact codes
      levels[k] = __ffma2_rn(make_float2(st[0], st[1]), cf, make_float2(zt[0], zt[1]));
    }
  }
#pragma unroll
  for (int i = 0; i < BITS; ++i) words[i] += odd[i];
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// In place: mn[0] = min and mx[0] = max of the N values, by passes of
// three-input operations (a pass maps N values to ceil(N / 3)).
template <int N>
__device__ __forceinline__ void reduce_min_max(float* mn, float* mx) {
  if constexpr (N > 1) {
    constexpr int M = (N + 2) / 3;
#pragma unroll
    for (int i = 0; i < M; ++i) {
      if (3 * i + 2 < N) {
        mn[i] = min3f(mn[3 * i], mn[3 * i + 1], mn[3 * i + 2]);
        mx[i] = max3f(mx[3 * i], mx[3 * i + 1], mx[3 * i + 2]);
      } else if (3 * i + 1 < N) {
        mn[i] = fminf(mn[3 * i], mn[3 * i + 1]);
        mx[i] = fmaxf(mx[3 * i], mx[3 * i + 1]);
      } else {
        mn[i] = mn[3 * i];
        mx[i] = mx[3 * i];
      }
    }
    reduce_min_max<M>(mn, mx);
  }
}

// Affine quantisation [RQ §2.1] of one lane's 32 values and the packed store;
// if `levels` is given it receives the stored levels fma(s~, code, z~) (what
// a reader of the record reconstructs).  Group parts: channels 0-15 (.x)
// and 16-31 (.y) for g = 16, the whole slice (or several lanes) otherwise.
template <int D, int BITS, int G>
__device__ __forceinline__ void quantize_store(const float2 (&v)[16], int slice, bool active,
                                               uint32_t* codes_row, unsigned char* meta_row,
                                               bool m16,
                                               float2* levels = nullptr) {
  constexpr uint32_t QMAX = (1u << BITS) - 1u;
  constexpr int NG = G < 32 ? 2 : 1;        // group parts per lane
  constexpr int LPG = G > 32 ? G / 32 : 1;  // lanes sharing a group
  float st[2], zt[2], inv[2], gmn[2], gmx[2];
  uint32_t metaw[2];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    // min / max as trees of three-input operations (exact in any order)
    float tn[16], tx[16];
    if constexpr (NG == 2) {
#pragma unroll
      for (int k = 0; k < 16; ++k) tn[k] = tx[k] = gi == 0 ? v[k].x : v[k].y;
      reduce_min_max<16>(tn, tx);
    } else {
      float un[32], ux[32];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        un[k] = ux[k] = v[k].x;
        un[k + 16] = ux[k + 16] = v[k].y;
      }
      reduce_min_max<32>(un, ux);
      tn[0] = un[0];
      tx[0] = ux[0];
    }
    float mn = tn[0], mx = tx[0];
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    mn = __fadd_rn(mn, 0.0f);   // a zero end of the range is +0
    mx = __fadd_rn(mx, 0.0f);
    gmn[gi] = mn;
    gmx[gi] = mx;
    const float s = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(QMAX));
    if (m16) {
      // 16-bit metadata: scale byte nearest to max(s, |mn| / 15.875), offset
      // byte = floor(8 mn / s~) clamped to int8, z~ = zq s~ / 8 (exact).
      const float s1 = __fdiv_rn(fabsf(mn), 15.875f);
      uint32_t sb = m16_scale_byte(s > s1 ? s : s1);
      st[gi] = m16_scale_value(sb);
      int zq = 0;
      if (st[gi] > 0.0f) {
        float tq = floorf(__fdiv_rn(__fmul_rn(8.0f, mn), st[gi]));
        // the offset byte would saturate: one scale step up (always enough)
        if ((tq < -128.0f || tq > 127.0f) && sb < 0xFFu) {
          ++sb;
          st[gi] = m16_scale_value(sb);
          tq = floorf(__fdiv_rn(__fmul_rn(8.0f, mn), st[gi]));
        }
        zq = tq < -128.0f ? -128 : (tq > 127.0f ? 127 : static_cast<int>(tq));
      }
      zt[gi] = __fmul_rn(__fmul_rn(static_cast<float>(zq), st[gi]), 0.125f);
      metaw[gi] = sb | ((static_cast<uint32_t>(zq) & 0xFFu) << 8);
    } else {
      const __half sh = __float2half_rn(s);
      const __half zh = __float2half_rn(mn);
      st[gi] = __half2float(sh);
      zt[gi] = __half2float(zh);
      metaw[gi] = static_cast<uint32_t>(__half_as_ushort(sh)) |
                  (static_cast<uint32_t>(__half_as_ushort(zh)) << 16);
    }
    inv[gi] = (st[gi] > 0.0f) ? __frcp_rn(st[gi]) : 0.0f;
  }
  // (x - z~) * (1/s~) is monotone in x: when both ends of every group of the
  // warp map into [-1/2, 2^b - 1/2), the upper clamp can change no code
  bool in_range = true;
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    const float ulo = __fmul_rn(__fsub_rn(gmn[gi], zt[gi]), inv[gi]);
    const float uhi = __fmul_rn(__fsub_rn(gmx[gi], zt[gi]), inv[gi]);
    in_range = in_range && ulo >= -0.5f && uhi < static_cast<float>(QMAX) + 0.5f;
  }
  const bool lower_only = __all_sync(0xffffffffu, in_range);
  if constexpr (NG == 1) {
    st[1] = st[0];
    zt[1] = zt[0];
    inv[1] = inv[0];
  }
  const float2 nz = make_float2(-zt[0], -zt[1]), iv = make_float2(inv[0], inv[1]);
  uint32_t words[BITS];
  if (levels == nullptr) {
    if (lower_only)
      pack_codes<BITS, 1, false>(v, nz, iv, st, zt, words, levels);
    else
      pack_codes<BITS, 2, false>(v, nz, iv, st, zt, words, levels);
  } else {
    if (lower_only)
      pack_codes<BITS, 1, true>(v, nz, iv, st, zt, words, levels);
    else
      pack_codes<BITS, 2, true>(v, nz, iv, st, zt, words, levels);
  }
  if (!active) return;
  uint32_t* cw = codes_row + slice * BITS;
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(cw) = make_uint4(words[0], words[1], words[2], words[3]);
  } else {
    *reinterpret_cast<uint2*>(cw) = make_uint2(words[0], words[1]);
  }
  if constexpr (NG == 2) {
    if (m16)
      reinterpret_cast<uint32_t*>(meta_row)[slice] = metaw[0] | (metaw[1] << 16);
    else
      reinterpret_cast<uint2*>(meta_row)[slice] = make_uint2(metaw[0], metaw[1]);
  } else if constexpr (LPG == 1) {
    if (m16)
      reinterpret_cast<uint16_t*>(meta_row)[slice] = static_cast<uint16_t>(metaw[0]);
    else
      reinterpret_cast<uint32_t*>(meta_row)[slice] = metaw[0];
  } else {
    if ((slice % LPG) == 0) {
      if (m16)
        reinterpret_cast<uint16_t*>(meta_row)[slice / LPG] = static_cast<uint16_t>(metaw[0]);
      else
        reinterpret_cast<uint32_t*>(meta_row)[slice / LPG] = metaw[0];
    }
  }
}

// Batch-head row and token of a flattened row index (32-bit division when
// every row index fits in 32 bits).
__device__ __forceinline__ void split_row(int64_t row, int32_t n, bool narrow, int64_t& bhi,
                                          int64_t& tn) {
  if (narrow) {
    const uint32_t r = static_cast<uint32_t>(row), q = r / static_cast<uint32_t>(n);
    bhi = q;
    tn = r - q * static_cast<uint32_t>(n);
  } else {
    bhi = row / n;
    tn = row - bhi * n;
  }
}

// Least-squares coefficient of z against the reference over the row
// [RQ §3.2 scaling coefficient, App. G.1]: alpha~ = bf16(<z, ref> / <ref, ref>)
// (0 for a zero reference; 1 without LS scaling); z becomes the residual
// fma(-alpha~, ref, z).  The dots run lane-serially in channel order, then
// across the row's lanes.
template <int D>
__device__ __forceinline__ __nv_bfloat16 ls_residual(float2 (&v)[16], const float2 (&ref)[16],
                                                     bool unit_alpha) {
  constexpr int P = D / 32;
  float a = 1.0f;
  if (!unit_alpha) {
    float dzr = 0.0f, drr = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float z = ch_of(v, k), r = ch_of(ref, k);
      dzr = __fmaf_rn(z, r, dzr);
      drr = __fmaf_rn(r, r, drr);
    }
#pragma unroll
    for (int off = P / 2; off >= 1; off >>= 1) {
      dzr = __fadd_rn(dzr, __shfl_xor_sync(0xffffffffu, dzr, off));
      drr = __fadd_rn(drr, __shfl_xor_sync(0xffffffffu, drr, off));
    }
    a = (drr > 0.0f) ? __fdiv_rn(dzr, drr) : 0.0f;
  }
  const __nv_bfloat16 ab = __float2bfloat16_rn(a);
  const float at = __bfloat162float(ab);
  const float2 na = make_float2(-at, -at);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __ffma2_rn(na, ref[k], v[k]);
  return ab;
}

// Row of bf16 x -> Z in one lane's 16 pairs: the Hadamard transform, or the
// dense rotation of the row's head (DENSE).
template <int D, bool DENSE>
__device__ __forceinline__ void load_input(const QuantParams& p, int64_t row, int64_t bhi,
                                           bool active, int lane, float* tile, float2 (&v)[16]) {
  if constexpr (DENSE) {
    uint4 q[4];
    if (active) {
      const uint4* src = reinterpret_cast<const uint4*>(p.x + row * D + (lane % (D / 32)) * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = src[i];
    }
    rotate_dense<D>(q, active, lane, static_cast<int>(bhi % p.heads), p.urot, tile, v);
  } else {
    load_rotate<D>(p.x + (active ? row : 0) * D, active, lane % (D / 32), p.rot_scale, v);
  }
}

template <int D, int BITS, int G, bool DENSE>
__global__ void __launch_bounds__(kQuantThreads, 2)
    quantize_kernel(const __grid_constant__ QuantParams p) {
  constexpr int P = D / 32;
  constexpr int RPW = 32 / P;
  const int lane = threadIdx.x & 31;
  const int slice = lane % P;
  const int64_t total = static_cast<int64_t>(p.bh) * p.n;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) +
                       (threadIdx.x >> 5);
  const bool narrow = total <= 0xFFFFFFFFll;
  float* tile = nullptr;
  if constexpr (DENSE) {
    __shared__ __align__(16) float dense_tile[kQuantThreads * kDenseLaneFloats];
    tile = dense_tile + threadIdx.x * kDenseLaneFloats;
  }
  for (int64_t base = warp * RPW; base < total; base += nwarps * RPW) {
    const int64_t row = base + lane / P;
    const bool active = row < total;
    int64_t bhi, tn;
    split_row(active ? row : 0, p.n, narrow, bhi, tn);
    const int64_t t = p.t0 + tn;
    float2 v[16];
    if (p.dst.has_alpha) {
      // The reference is rebuilt from the cache first (its temporaries are
      // dead before the input row is loaded).  Fixed mean removed from the
      // input [RQ App. G.2]; least-squares coefficient against the
      // reconstructed reference [RQ §3.2 scaling coefficient, App. G.1],
      // then the residual.
      float2 ref[16];
      if (active) {
        chain_slice(p.ref, p.nref, bhi, p.nblk, t, slice, D, ref);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) ref[k] = make_float2(0.0f, 0.0f);
      }
      load_input<D, DENSE>(p, row, bhi, active, lane, tile, v);
      if (p.dst.mean != nullptr && active) sub_mean(p.dst, bhi, slice, D, v);
      const __nv_bfloat16 ab = ls_residual<D>(v, ref, p.unit_alpha != 0);
      if (active && slice == 0)
        *rec_alpha(comp_record(p.dst, bhi, p.nblk, t), D, BITS, G, static_cast<int>(t % kBlock),
                   p.dst.meta16 ? 2 : 4) =
            __bfloat16_as_ushort(ab);
    } else {
      load_input<D, DENSE>(p, row, bhi, active, lane, tile, v);
    }
    unsigned char* rec = comp_record(p.dst, bhi, p.nblk, t);
    const int i = static_cast<int>(t % kBlock);
    unsigned char* mrow = p.dst.meta16
                              ? reinterpret_cast<unsigned char*>(rec_meta16(rec, D, BITS, G, i))
                              : reinterpret_cast<unsigned char*>(rec_meta(rec, D, BITS, G, i));
    quantize_store<D, BITS, G>(v, slice, active, rec_codes(rec, D, BITS, i), mrow,
                               p.dst.meta16 != 0);
  }
}

// Record of component c at token t of row `row`, geometry fixed at compile
// time: codes, metadata and (residual loops) the LS coefficient's slot.
template <int D, int BITS, int G>
__device__ __forceinline__ void quantize_at(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                            const float2 (&v)[16], int slice, bool active,
                                            float2* levels, int alpha_bits) {
  constexpr int CW = D * BITS / 32;   // code words per token
  unsigned char* rec = comp_record(c, row, nblk, t);
  const int i = static_cast<int>(t % kBlock);
  const bool m16 = c.meta16 != 0;
  const int mb = m16 ? 2 : 4;
  uint32_t* cw = reinterpret_cast<uint32_t*>(rec) + i * CW;
  unsigned char* mw = rec + kBlock * 4 * CW + i * (D / G) * mb;
  if (alpha_bits >= 0 && active && slice == 0)
    reinterpret_cast<uint16_t*>(rec + kBlock * (4 * CW + mb * (D / G)))[i] =
        static_cast<uint16_t>(alpha_bits);
  quantize_store<D, BITS, G>(v, slice, active, cw, mw, m16, levels);
}

// Quantisation of one component at token t (run-time bits / group): codes,
// metadata, the LS coefficient's bf16 bits when alpha_bits >= 0, and (if
// `levels`) the stored levels of this lane's 32 channels.
template <int D>
__device__ __forceinline__ void quantize_comp(const Comp& c, int64_t row, int64_t nblk, int64_t t,
                                              const float2 (&v)[16], int slice, bool active,
                                              float2* levels, int alpha_bits = -1) {
  const int key = c.bits * 1000 + c.group;
  switch (key) {
    case 2016: quantize_at<D, 2, 16>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    case 2032: quantize_at<D, 2, 32>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    case 2064: quantize_at<D, 2, 64>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    case 4016: quantize_at<D, 4, 16>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    case 4032: quantize_at<D, 4, 32>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    case 4064: quantize_at<D, 4, 64>(c, row, nblk, t, v, slice, active, levels, alpha_bits); break;
    default:
      if constexpr (D >= 128) {
        if (key == 2128)
          quantize_at<D, 2, 128>(c, row, nblk, t, v, slice, active, levels, alpha_bits);
        else if (key == 4128)
          quantize_at<D, 4, 128>(c, row, nblk, t, v, slice, active, levels, alpha_bits);
      }
      break;
  }
}

// Every loop of a (layer, token range) for one side (blockIdx.y): the anchor
// is quantised first and its stored levels stay in registers as the
// reference; each other loop then takes its LS coefficient, residual and
// quantisation against it [RQ §3.2, §3.4, App. G.1].  Loops run away from
// the anchor (p.order); under a chained policy the reference becomes
// Z^_r = fma(alpha~_r, Z^_ref, D(c_r)) after loop r.  The anchor is read
// once and never re-read from the cache; the arithmetic (and so every
// stored bit) is that of the per-loop kernels.
// The fused kernel's dense instantiation keeps two ring slots per warp and a
// CTA copy of the current head's matrix.
template <bool DENSE>
constexpr int loops_stages() { return DENSE ? 2 : kQStages; }
template <bool DENSE>
constexpr int loops_smem() {
  return (kQuantThreads / 32) * loops_stages<DENSE>() * kQSlotBytes +
         (DENSE ? kDenseTileBytes + kUshBytes : 0);
}

template <int D, bool CHAINED, bool DENSE>
__global__ void __launch_bounds__(kQuantThreads, 2)
    quantize_loops_kernel(const __grid_constant__ QuantLoopsParams p) {
  constexpr int P = D / 32;
  constexpr int RPW = 32 / P;
  constexpr int NS = loops_stages<DENSE>();
  static_assert(RPW * D * 2 == kQSlotBytes, "a slot holds one job of RPW rows");
  extern __shared__ __align__(128) unsigned char qsmem[];
  const int side = blockIdx.y;
  const uint16_t* xs = p.x[side];
  if (xs == nullptr) return;
  const int lane = threadIdx.x & 31;
  const int slice = lane % P;
  const int64_t total = static_cast<int64_t>(p.bh) * p.n;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) +
                       (threadIdx.x >> 5);
  const int a = p.anchor;
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(qsmem)) +
                        (threadIdx.x >> 5) * (NS * kQSlotBytes);
  // Job j of this warp: rows base_j .. base_j + RPW - 1 of loop li_j (li 0 is
  // the anchor, li k >= 1 is p.order[k - 1]); jobs run row group by row
  // group, every loop of a group in turn.
  int64_t is_base = warp * RPW;
  int is_li = 0, is_slot = 0;
  auto issue_next = [&]() {
    if (is_base < total) {
      const int r = is_li == 0 ? a : p.order[is_li - 1];
      const int64_t left = total - is_base;
      stage_rows<D>(ring + is_slot * kQSlotBytes,
                    reinterpret_cast<const unsigned char*>(
                        xs + (static_cast<int64_t>(r) * total + is_base) * D),
                    left < RPW ? static_cast<int>(left) : RPW, lane);
    }
    cp_async_commit();   // one group per job, empty past the end
    if (++is_li == p.nloops) {
      is_li = 0;
      is_base += nwarps * RPW;
    }
    is_slot = is_slot + 1 == NS ? 0 : is_slot + 1;
  };
#pragma unroll
  for (int s = 0; s + 1 < NS; ++s) issue_next();
  int slot = 0;
  // the job in `slot` has landed (this lane's copies, then the warp's); the
  // slot read in the previous job is free again and takes the next issue
  // dense: the CTA's shared matrix (head ush_head, -1 when the CTA's rows of
  // this pass span several heads)
  const uint32_t ush = static_cast<uint32_t>(__cvta_generic_to_shared(qsmem)) +
                       (kQuantThreads / 32) * NS * kQSlotBytes + (DENSE ? kDenseTileBytes : 0);
  int ush_head = -1;
  auto next_input = [&](bool active, int head, float2 (&v)[16]) {
    cp_async_wait<NS - 2>();
    __syncwarp();
    issue_next();
    uint4 q[4];
    read_slot<D>(ring + slot * kQSlotBytes, lane, q);
    slot = slot + 1 == NS ? 0 : slot + 1;
    if constexpr (DENSE)
      rotate_dense<D>(q, active, lane, head, p.urot[side],
                      reinterpret_cast<float*>(qsmem + (kQuantThreads / 32) * NS *
                                                           kQSlotBytes) +
                          threadIdx.x * kDenseLaneFloats,
                      v, ush, ush_head);
    else
      rotate_pieces<D>(q, active, slice, p.rot_scale, v);
  };
  const bool narrow = total <= 0xFFFFFFFFll;
  // CTA-uniform passes: every warp of the CTA takes part in each pass (its
  // rows may lie past the end), so the dense form can share one matrix
  constexpr int64_t kCtaRows = (kQuantThreads / 32) * RPW;
  for (int64_t cbase = static_cast<int64_t>(blockIdx.x) * kCtaRows; cbase < total;
       cbase += nwarps * RPW) {
    const int64_t base = cbase + (threadIdx.x >> 5) * RPW;
    if constexpr (DENSE) {
      __syncthreads();   // the previous pass is done with the shared matrix
      const int64_t last = (cbase + kCtaRows < total ? cbase + kCtaRows : total) - 1;
      const int64_t b0 = cbase / p.n, b1 = last / p.n;
      ush_head = b0 == b1 ? static_cast<int>(b0 % p.heads) : -1;
      if (ush_head >= 0) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.urot[side] + static_cast<size_t>(ush_head) * D * D);
        for (int c = threadIdx.x; c < D * D / 8; c += kQuantThreads) {
          const uint4 w = __ldg(src + c);
          const uint32_t dst = ush + ((c >> 4) * kUshStride + (c & 15) * 8) * 2;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w.x),
                       "r"(w.y), "r"(w.z), "r"(w.w)
                       : "memory");
        }
      }
      __syncthreads();
    }
    if (base >= total) continue;
    const int64_t row = base + lane / P;
    const bool active = row < total;
    int64_t bhi, tn;
    split_row(active ? row : 0, p.n, narrow, bhi, tn);
    const int64_t t = p.t0 + tn;
    const int head = static_cast<int>(bhi % p.heads);
    float2 ref[16], v[16];
    next_input(active, head, v);
    quantize_comp<D>(p.dst[side][a], bhi, p.nblk, t, v, slice, active, ref);
    for (int k = 0; k + 1 < p.nloops; ++k) {
      const int r = p.order[k];
      const Comp& c = p.dst[side][r];
      next_input(active, head, v);
      if (c.mean != nullptr && active) sub_mean(c, bhi, slice, D, v);
      const __nv_bfloat16 ab = ls_residual<D>(v, ref, p.unit_alpha != 0);
      float2 lv[16];   // stored levels, the next reference of a chain
      quantize_comp<D>(c, bhi, p.nblk, t, v, slice, active, CHAINED ? lv : nullptr,
                       __bfloat16_as_ushort(ab));
      if constexpr (CHAINED) {
        const float at = __bfloat162float(ab);
        const float2 a2 = make_float2(at, at);
#pragma unroll
        for (int j = 0; j < 16; ++j) ref[j] = __ffma2_rn(a2, ref[j], lv[j]);
        if (c.mean != nullptr && active) add_mean(c, bhi, slice, D, ref);
      }
    }
  }
  cp_async_wait<0>();   // nothing left in flight into the ring at exit
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
    float2 v[16];
    if (active) {
      chain_slice(p.comp, p.ncomp, row / p.n, p.nblk, p.t0 + row % p.n, slice, D, v);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = make_float2(0.0f, 0.0f);
    }
    if (p.urot != nullptr) {
      // X^ = U^T Z^ [RQ App. G.2]: the row through shared memory, fp32 sums
      // over j ascending, lane `slice` writing channels [32 slice, +32).
      if constexpr (D == 128) {
        __shared__ float zrow[kQuantThreads / 32][RPW][D];
        float* zr = zrow[threadIdx.x >> 5][lane / P];
#pragma unroll
        for (int k = 0; k < 32; ++k) zr[slice * 32 + k] = ch_of(v, k);
        __syncwarp();
        float o[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0.0f;
        const uint16_t* uh = p.urot + static_cast<size_t>(active ? (row / p.n) % p.heads : 0) *
                                          D * D + slice * 32;
        for (int j = 0; j < D; ++j) {
          const float zj = zr[j];
          const uint4* up = reinterpret_cast<const uint4*>(uh + static_cast<size_t>(j) * D);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = __ldg(up + i);
            const uint32_t hw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 u = __half22float2(*reinterpret_cast<const __half2*>(&hw[e]));
              o[8 * i + 2 * e] = fmaf(u.x, zj, o[8 * i + 2 * e]);
              o[8 * i + 2 * e + 1] = fmaf(u.y, zj, o[8 * i + 2 * e + 1]);
            }
          }
        }
        __syncwarp();
        if (active) {
          float4* dst = reinterpret_cast<float4*>(p.out + row * D + slice * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
      continue;
    }
    // X^ = H^T Z^ = H Z^ (the normalised Sylvester matrix is symmetric).
    fwht_row<D>(v, slice);
    if (active) {
      const float rs = p.rot_scale;
      float4* dst = reinterpret_cast<float4*>(p.out + row * D + slice * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(ch_of(v, 4 * i) * rs, ch_of(v, 4 * i + 1) * rs,
                             ch_of(v, 4 * i + 2) * rs, ch_of(v, 4 * i + 3) * rs);
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
  if (p.urot != nullptr) {
    if constexpr (D == 128)
      quantize_kernel<D, BITS, G, true><<<grid, kQuantThreads, 0, s>>>(p);
    else
      return cudaErrorInvalidValue;
  } else {
    quantize_kernel<D, BITS, G, false><<<grid, kQuantThreads, 0, s>>>(p);
  }
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

template <int D, bool CHAINED, bool DENSE>
cudaError_t launch_loops_t(const QuantLoopsParams& p, dim3 grid, cudaStream_t s) {
  constexpr int smem = loops_smem<DENSE>();
  const cudaError_t e = cudaFuncSetAttribute(quantize_loops_kernel<D, CHAINED, DENSE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  quantize_loops_kernel<D, CHAINED, DENSE><<<grid, kQuantThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// Both sides of a fused call use the same transform kind (a cache sets its
// K and V rotations together or not at all on a side: a side without one
// keeps the Hadamard transform and runs in a second launch).
template <int D, bool CHAINED>
cudaError_t launch_loops(const QuantLoopsParams& p, dim3 grid, cudaStream_t s) {
  const bool dk = p.urot[0] != nullptr && p.x[0] != nullptr;
  const bool dv = p.urot[1] != nullptr && p.x[1] != nullptr;
  if (!dk && !dv) return launch_loops_t<D, CHAINED, false>(p, grid, s);
  if constexpr (D != 128) {
    return cudaErrorInvalidValue;
  } else {
    // one launch per transform kind; a side of the other kind is skipped
    QuantLoopsParams pd = p, ph = p;
    pd.x[0] = dk ? p.x[0] : nullptr;
    pd.x[1] = dv ? p.x[1] : nullptr;
    ph.x[0] = dk ? nullptr : p.x[0];
    ph.x[1] = dv ? nullptr : p.x[1];
    cudaError_t e = launch_loops_t<D, CHAINED, true>(pd, grid, s);
    if (e == cudaSuccess && (ph.x[0] != nullptr || ph.x[1] != nullptr))
      e = launch_loops_t<D, CHAINED, false>(ph, grid, s);
    return e;
  }
}

cudaError_t launch_quantize_loops(const QuantLoopsParams& p, int D, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.bh) * p.n;
  if (rows == 0) return cudaSuccess;
  const dim3 grid(quant_grid(rows, D), 2);
  if (D == 64) return p.chained ? launch_loops<64, true>(p, grid, s) : launch_loops<64, false>(p, grid, s);
  if (D == 128) return p.chained ? launch_loops<128, true>(p, grid, s) : launch_loops<128, false>(p, grid, s);
  return cudaErrorInvalidValue;
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
