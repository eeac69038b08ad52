// rq_internal.cuh -- device helpers and kernel parameter blocks shared by the
// librq translation units (never installed; the public ABI is librq.h).
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "librq.h"

namespace rq {

// Device-side error bits recorded in the decode workspace.
constexpr uint32_t kErrSeqLen = 1u;    // a seq_lens entry was outside [0, max_seq_len]
constexpr uint32_t kErrTimeout = 2u;   // a bounded mbarrier wait ran out
constexpr uint32_t kErrRange = 4u;     // a value weight left the scaled-accumulator range

// Tokens per pipeline stage of the generic decode kernel (two records).
constexpr int kChunk = 64;
constexpr int kDecodeThreads = 128;

// ---------------------------------------------------------------------------
// Parameter blocks
// ---------------------------------------------------------------------------

// One packed component (anchor or one residual loop) of one side, stored as
// 32-token records [codes[32][D*bits/32] | meta[32][D/group] | alpha[32]].
struct Comp {
  unsigned char* base;     // record of (row 0, block 0)
  uint32_t rec_bytes;      // bytes per record
  int32_t bits;
  int32_t group;
  int32_t has_alpha;       // 0 for the anchor
  int32_t meta16;          // 1: 16-bit metadata per group (scale byte | offset byte)
  // Fixed mean of this residual loop [RQ App. G.2]: fp32 [kv_heads][D] in
  // the rotated domain (row b*H + h uses row h), or nullptr.
  const float* mean;
  int32_t heads;
};

constexpr int kBlock = RQ_BLOCK_TOKENS;
// Rows hold a multiple of 64 tokens, so a 64-token stage aligned to 64 never
// leaves its row.
constexpr int kRowTokens = 64;
static_assert(kChunk % kBlock == 0 && kRowTokens % kChunk == 0, "stages are whole records");

// Record holding token t of row `row` (nblk = records per row).
__host__ __device__ inline unsigned char* comp_record(const Comp& c, int64_t row, int64_t nblk,
                                                      int64_t t) {
  return c.base + (row * nblk + t / kBlock) * static_cast<int64_t>(c.rec_bytes);
}
__host__ __device__ inline uint32_t* rec_codes(unsigned char* rec, int D, int bits, int i) {
  return reinterpret_cast<uint32_t*>(rec) + i * (D * bits / 32);
}
__host__ __device__ inline uint32_t* rec_meta(unsigned char* rec, int D, int bits, int group,
                                              int i) {
  return reinterpret_cast<uint32_t*>(rec) + kBlock * (D * bits / 32) + i * (D / group);
}
// 16-bit metadata form: meta16 [32][D/group] after the codes.
__host__ __device__ inline uint16_t* rec_meta16(unsigned char* rec, int D, int bits, int group,
                                                int i) {
  return reinterpret_cast<uint16_t*>(rec + kBlock * 4 * (D * bits / 32)) + i * (D / group);
}
// meta_bytes: 4 (fp16 scale | fp16 offset) or 2 (16-bit metadata).
__host__ __device__ inline uint16_t* rec_alpha(unsigned char* rec, int D, int bits, int group,
                                               int i, int meta_bytes = 4) {
  return reinterpret_cast<uint16_t*>(rec + kBlock * (4 * (D * bits / 32) +
                                                     meta_bytes * (D / group))) + i;
}

// 16-bit metadata: the scale byte is unsigned e5m3 with this exponent bias
// (byte 8E + m -> (1 + m/8) 2^(E - bias), E = 0 -> 0).
constexpr int kM16Bias = 18;

// Scale byte nearest to s > 0 (ties to even m); below the range -> the
// smallest positive value, above it -> the largest; s <= 0 or NaN -> 0.
__host__ __device__ inline uint32_t m16_scale_byte(float s) {
  if (!(s > 0.0f)) return 0u;
  uint32_t b;
  memcpy(&b, &s, sizeof(b));
  int E = static_cast<int>((b >> 23) & 0xFFu);
  if (E == 0xFF) return 0xFFu;
  if (E == 0) return 0x08u;
  uint32_t m = (b & 0x7FFFFFu) >> 20;
  const uint32_t rem = b & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (m & 1u))) ++m;
  if (m == 8u) {
    m = 0u;
    ++E;
  }
  const int Eb = E - 127 + kM16Bias;
  if (Eb < 1) return 0x08u;
  if (Eb > 31) return 0xFFu;
  return (static_cast<uint32_t>(Eb) << 3) | m;
}

// Offset of a 16-bit metadata word given its scale: zq * s~ / 8 (exact).
__host__ __device__ inline float m16_offset(uint32_t h, float s) {
  return static_cast<float>(static_cast<int8_t>(static_cast<uint8_t>(h >> 8))) * s * 0.125f;
}

// Value of a scale byte (exact: the byte's fields go straight into the
// exponent and the top mantissa bits).
__host__ __device__ inline float m16_scale_value(uint32_t byte) {
  const uint32_t Eb = (byte >> 3) & 31u;
  const uint32_t bits = Eb == 0u ? 0u : (((Eb + 127u - kM16Bias) << 23) | ((byte & 7u) << 20));
  float f;
  memcpy(&f, &bits, sizeof(f));
  return f;
}

struct QuantParams {
  int32_t unit_alpha;      // 1: alpha = 1 (no LS scaling)
  const uint16_t* x;       // bf16 [B*H][n][D]
  int32_t bh;              // B*H
  int32_t n;
  int32_t t0;
  int64_t nblk;            // records per row
  Comp dst;                // destination component
  // Reference chain, nearest first: for a shared anchor one entry (the
  // anchor); for a chain the neighbour toward the anchor first, the anchor
  // last.
  int32_t nref;
  Comp ref[RQ_MAX_LOOPS];
  float rot_scale;         // fp32(1/sqrt(D))
  // Dense rotation of this (layer, side): binary16 [heads][D][D], or nullptr
  // for the Hadamard transform.
  const uint16_t* urot;
  int32_t heads;
};

// Every loop of one (layer, token range), both sides, in one launch.
struct QuantLoopsParams {
  const uint16_t* x[2];    // bf16 [L][B*H][n][D] per side (K, V); nullptr skips the side
  int32_t bh, n, nloops;
  int32_t anchor;          // anchor loop
  int32_t order[RQ_MAX_LOOPS];   // the other loops, away from the anchor
  int32_t chained;         // 1: loop order[k] references order[k-1] (the anchor for k = 0)
  int32_t unit_alpha;      // 1: alpha = 1 (no LS scaling)
  int64_t t0, nblk;
  Comp dst[2][RQ_MAX_LOOPS];
  float rot_scale;
  const uint16_t* urot[2]; // dense rotations per side (binary16 [heads][D][D]) or nullptr
  int32_t heads;
};

struct DequantParams {
  int32_t bh, n, t0;
  int64_t nblk;
  int32_t ncomp;           // chain: [0] = the loop itself ... [ncomp-1] = anchor
  Comp comp[RQ_MAX_LOOPS];
  float rot_scale;
  float* out;              // fp32 [B*H][n][D]
  const uint16_t* urot;    // dense rotation (binary16 [heads][D][D]) or nullptr
  int32_t heads;
};

struct DecodeParams {
  int32_t bh;              // B*H
  int32_t heads;
  int64_t nblk;            // records per row
  int32_t ncomp;           // [0] = the loop's own residual ... [ncomp-1] = anchor
  Comp k[RQ_MAX_LOOPS];
  Comp v[RQ_MAX_LOOPS];
  const uint16_t* q;       // bf16 [B*H][D]
  const uint16_t* kcur;
  const uint16_t* vcur;
  const int32_t* seq_lens; // [B]
  int32_t max_seq_len;
  float scale_log2;        // softmax scale * log2(e)
  float rot_scale;
  float* out;              // fp32 [B*H][D]
  // workspace
  float* partials;         // [B*H][splits][D+2]
  uint32_t* counters;      // [B*H]
  uint32_t* err;           // [1]
  int32_t splits;
  int32_t chunk;           // tokens per pipeline stage (whole records)
  int32_t chunks_per_split;
  int32_t stages;
  uint32_t stage_bytes;
  int32_t use_fast;        // warp-specialised kernel for a compiled layout
  // Dense rotations of the layer (binary16 [heads][D][D]) or nullptr for the
  // Hadamard transform.
  const uint16_t* urot_k;
  const uint16_t* urot_v;
};

struct DecodeBf16Params {
  int32_t bh, heads;
  int64_t tstride;
  const uint16_t* k;       // bf16 [B*H][tstride][D]
  const uint16_t* v;
  const uint16_t* q;
  const uint16_t* kcur;
  const uint16_t* vcur;
  const int32_t* seq_lens;
  int32_t max_seq_len;
  float scale_log2;
  float* out;
  float* partials;
  uint32_t* counters;
  uint32_t* err;
  int32_t splits;
  int32_t chunks_per_split;
  int32_t stages;
  uint32_t stage_bytes;
};

// ---------------------------------------------------------------------------
// Host-side launchers (defined in the .cu files)
// ---------------------------------------------------------------------------

// Self-test: one CTA waits `limit_ns` on an mbarrier phase nothing completes.
cudaError_t launch_selftest_wait(uint32_t* err, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_quantize(const QuantParams& p, int D, int bits, int group,
                            cudaStream_t s);
cudaError_t launch_dequantize(const DequantParams& p, int D, cudaStream_t s);
cudaError_t launch_quantize_loops(const QuantLoopsParams& p, int D, cudaStream_t s);
// generic compressed decode (any chain of bits / groups), chunk kChunk
cudaError_t launch_decode(const DecodeParams& p, int D, cudaStream_t s);
// decode for compiled layouts: stages, tokens per stage and resident CTAs
bool fast_decode_plan(const DecodeParams& p, int D, int* stages, int* chunk, int* ctas_per_sm);
cudaError_t launch_decode_fast(const DecodeParams& p, int D, cudaStream_t s);
// uncompressed bf16 decode, chunk bf16_chunk(D)
cudaError_t launch_decode_bf16(const DecodeBf16Params& p, int D,
                               cudaStream_t s);
uint32_t bf16_stage_bytes(int D);
int bf16_chunk(int D);
cudaError_t bf16_occupancy(int D, int stages, int* occ);
// bytes of one pipeline stage for a decode call
uint32_t decode_stage_bytes(const DecodeParams& p, int D);
// dynamic shared memory of a decode launch (stage ring or merge scratch)
size_t decode_dyn_smem(int D, int stages, uint32_t stage_bytes);
// resident CTAs per SM of the generic decode kernel at this dynamic shared memory
cudaError_t decode_occupancy(int D, size_t dyn_smem, int* ctas_per_sm);

// Host planning of a compressed decode call (pointers into the workspace are
// left for the caller to set): component chain, kernel choice, stages, splits.
rq_status plan_decode(const rq_cache* c, int32_t layer, int32_t loop, int32_t max_seq_len,
                      DecodeParams* p, int* D);
float decode_scale_log2(float softmax_scale, int D);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------

// Storage order of packed codes.  A lane's 32-channel slice of a row starts
// at word slice*BITS; inside it channel ch (0..31) sits at
//   BITS = 2: word ch/16, bits 2*(ch%16)
//   BITS = 4: word 2*(ch/16) + ((ch%16 >> 1) & 1), nibble 2*((ch%16) >> 2) + (ch & 1)
// so that, for both widths, masking bytes of the words yields the channel
// quads {s, s+4, s+8, s+12} of each 16-channel block.
template <int BITS>
__host__ __device__ constexpr int slice_word(int ch) {
  return BITS == 2 ? ch / 16 : 2 * (ch / 16) + (((ch % 16) >> 1) & 1);
}
template <int BITS>
__host__ __device__ constexpr int slice_shift(int ch) {
  return BITS == 2 ? 2 * (ch % 16) : 4 * (2 * ((ch % 16) >> 2) + (ch & 1));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 16);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on a phase of an mbarrier: gives up once `limit_ns` of device
// time have passed (checked every 64 polls), or after 2^26 polls whatever the
// clock says, records kErrTimeout and returns false.
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  uint64_t t0 = 0;
  for (uint32_t it = 0; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (it == 0) t0 = global_ns();   // the clock is read only once a wait is needed
    if (it > 16) __nanosleep(256);
    if ((it & 63u) == 63u && global_ns() - t0 > limit_ns) break;
  }
  atomicOr(err, kErrTimeout);
  return false;
}

// Bulk (non-tensor) asynchronous copy global -> this CTA's shared memory,
// completing `bytes` of transaction count on `bar`.  No multicast.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src,
                                              uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace rq
