// rq_noalloc.cu -- decode attention for callers that cannot allocate device
// memory (for example code running inside a host framework that owns every
// allocation, or a tight serving loop that may not call cudaMalloc): the
// split-K scratch lives in a fixed-size array of this module instead of a
// caller-provided workspace.
#include <math.h>
#include <string.h>

#include <mutex>

#include "rq_internal.cuh"

namespace {

using namespace rq;

// Scratch of rq_decode_attention_noalloc: [error word | split counters |
// split partials].  8 MiB, held by every device that loads the library until
// the process exits.  The counters have a fixed region for the largest
// batch * kv_heads a layout allows, so the partials of one call never land on
// the counters of a later call with more rows (the counters must start at
// zero; the kernels return every counter they use to zero).
constexpr size_t kNoAllocScratchBytes = 8u << 20;
constexpr size_t kHeaderAlign = 256;
constexpr size_t kMaxRows = 65535;   // batch * kv_heads limit of rq_layout_validate

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices];   // device address of g_decode_scratch, per device

// Device address of the scratch for the current device.  The first call on a
// device looks the address up (cudaGetSymbolAddress, with that device
// current) and zeroes the array once; the kernels leave the split counters at
// zero after every call.
rq_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
      return RQ_ERR_CUDA;
    if (cudaMemset(ptr, 0, kNoAllocScratchBytes) != cudaSuccess) return RQ_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return RQ_OK;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" rq_status rq_decode_attention_noalloc(const rq_cache* c, int32_t layer, int32_t loop,
                                                 const void* q, const int32_t* seq_lens,
                                                 int32_t max_seq_len, const void* k_cur,
                                                 const void* v_cur, float softmax_scale,
                                                 float* out, void* stream) {
  if (c == nullptr || c->k_base == nullptr || c->v_base == nullptr) return RQ_ERR_INVALID_ARG;
  if (rq_layout_validate(&c->layout) != RQ_OK) return RQ_ERR_INVALID_ARG;
  const rq_layout& l = c->layout;
  if (layer < 0 || layer >= l.num_layers || loop < 0 || loop >= l.num_loops)
    return RQ_ERR_INVALID_ARG;
  if (q == nullptr || seq_lens == nullptr || k_cur == nullptr || v_cur == nullptr ||
      out == nullptr)
    return RQ_ERR_INVALID_ARG;
  if (max_seq_len < 0) return RQ_ERR_INVALID_ARG;
  if (max_seq_len > l.max_tokens) return RQ_ERR_CAPACITY;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return RQ_ERR_INVALID_ARG;

  DecodeParams p;
  int D = 0;
  rq_status st = plan_decode(c, layer, loop, max_seq_len, &p, &D);
  if (st != RQ_OK) return st;

  // Fit the split partials into the fixed scratch: fewer splits if needed,
  // an error if even one split per (batch, head) does not fit.
  const size_t counters_off = kHeaderAlign;
  const size_t partials_off = align_up(counters_off + kMaxRows * 4, kHeaderAlign);
  const size_t per_split = static_cast<size_t>(p.bh) * (D + 2) * sizeof(float);
  if (partials_off + per_split > kNoAllocScratchBytes) return RQ_ERR_WORKSPACE;
  const int fit = static_cast<int>((kNoAllocScratchBytes - partials_off) / per_split);
  if (p.splits > fit) {
    const int chunks = (max_seq_len + p.chunk - 1) / p.chunk;
    int cps = (chunks + fit - 1) / fit;
    if (cps < 1) cps = 1;
    p.chunks_per_split = cps;
    p.splits = chunks > 0 ? (chunks + cps - 1) / cps : 1;
  }

  void* base = nullptr;
  if ((st = scratch_address(&base)) != RQ_OK) return st;
  unsigned char* scratch = static_cast<unsigned char*>(base);
  p.q = static_cast<const uint16_t*>(q);
  p.kcur = static_cast<const uint16_t*>(k_cur);
  p.vcur = static_cast<const uint16_t*>(v_cur);
  p.seq_lens = seq_lens;
  p.scale_log2 = decode_scale_log2(softmax_scale, D);
  p.out = out;
  p.err = reinterpret_cast<uint32_t*>(scratch);
  p.counters = reinterpret_cast<uint32_t*>(scratch + counters_off);
  p.partials = reinterpret_cast<float*>(scratch + partials_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = p.use_fast ? launch_decode_fast(p, D, s) : launch_decode(p, D, s);
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}
