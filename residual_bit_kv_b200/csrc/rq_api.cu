// rq_api.cu -- host side of the librq C ABI: argument validation, storage
// layout, split-K sizing and kernel launches.  See include/librq.h.
//
// Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
// Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
#include <math.h>
#include <string.h>

#include "rq_internal.cuh"

namespace {

using namespace rq;

constexpr uint64_t kAlign = 256;
constexpr int kMaxSplits = 1024;
constexpr int kMaxStages = 4;
constexpr double kCtaOverheadChunks = 4.0;   // per-CTA fixed cost, in chunk times
constexpr size_t kRingBudget = 100 * 1024;   // stage ring per CTA: two or more CTAs per SM

inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

inline bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

inline rq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Anchor loop of a layout: the final loop (Last-/Next-loop) or the first
// (First-/Previous-loop) [RQ §3.2, App. D].
inline int anchor_of(const rq_layout* l) {
  return (l->policy == RQ_POLICY_FIRST_LOOP || l->policy == RQ_POLICY_PREVIOUS_LOOP)
             ? 0
             : l->num_loops - 1;
}

inline bool chained_of(const rq_layout* l) {
  return l->policy == RQ_POLICY_NEXT_LOOP || l->policy == RQ_POLICY_PREVIOUS_LOOP;
}

// The loop that loop r references (r != anchor).
inline int reference_of(const rq_layout* l, int r) {
  if (l->policy == RQ_POLICY_NEXT_LOOP) return r + 1;
  if (l->policy == RQ_POLICY_PREVIOUS_LOOP) return r - 1;
  return anchor_of(l);
}

inline int64_t token_stride_of(const rq_layout* l) {
  return static_cast<int64_t>(align_up(static_cast<uint64_t>(l->max_tokens), kRowTokens));
}

inline int meta_bytes_of(const rq_layout* l) { return (l->flags & RQ_FLAG_META16) ? 2 : 4; }

inline uint32_t record_bytes(const rq_layout* l, int r) {
  const int D = l->head_dim;
  const uint32_t per_token = (D * l->bits[r] / 32) * 4 + (D / l->group[r]) * meta_bytes_of(l) +
                             (r != anchor_of(l) ? 2 : 0);
  return kBlock * per_token;   // a multiple of 64 bytes
}

// Byte offset of every component's first record inside one (layer, side);
// returns the layer bytes.  Anchor first, then the other loops ascending.
uint64_t layout_offsets(const rq_layout* l, uint64_t* comp_off, uint32_t* rec_bytes) {
  const uint64_t records = static_cast<uint64_t>(l->batch) * l->kv_heads *
                           (token_stride_of(l) / kBlock);
  const int L = l->num_loops;
  uint64_t off = 0;
  const int a = anchor_of(l);
  for (int k = 0; k < L; ++k) {
    const int r = (k == 0) ? a : (k - 1 < a ? k - 1 : k);
    comp_off[r] = off;
    rec_bytes[r] = record_bytes(l, r);
    off = align_up(off + records * rec_bytes[r], kAlign);
  }
  return off;
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return sms > 0 ? sms : 148;
}

int chunks_of(int32_t max_seq_len) { return (max_seq_len + kChunk - 1) / kChunk; }

int max_splits_of(int32_t max_seq_len) {
  int c = chunks_of(max_seq_len);
  if (c < 1) c = 1;
  return c > kMaxSplits ? kMaxSplits : c;
}

// Split count for a grid of bh * splits CTAs, each streaming `cps` chunks.
// Time model: (waves of resident CTAs) x (chunks per CTA + a fixed per-CTA
// cost of set-up, first-chunk latency and merge); splits start at
// the count that fills every resident slot once, so a small batch still
// occupies the whole GPU.  Splits never exceed max_splits_of() (the
// workspace bound) and never leave an empty split.
void choose_splits_on(int bh, int32_t max_seq_len, int chunk, int ctas_per_sm, int sms,
                      int* splits, int* cps);

void choose_splits(int bh, int32_t max_seq_len, int chunk, int ctas_per_sm, int* splits,
                   int* cps) {
  choose_splits_on(bh, max_seq_len, chunk, ctas_per_sm, device_sms(), splits, cps);
}

// The plan for a device with `sms` multiprocessors (host logic only).
void choose_splits_on(int bh, int32_t max_seq_len, int chunk, int ctas_per_sm, int sms,
                      int* splits, int* cps) {
  const int chunks = (max_seq_len + chunk - 1) / chunk;
  if (chunks == 0) {
    *splits = 1;
    *cps = 0;
    return;
  }
  const int64_t slots = static_cast<int64_t>(sms > 0 ? sms : 1) * (ctas_per_sm > 0 ? ctas_per_sm : 1);
  int smax = max_splits_of(max_seq_len);
  if (smax > chunks) smax = chunks;
  int smin = static_cast<int>((slots + bh - 1) / bh);
  if (smin > smax) smin = smax;
  if (smin < 1) smin = 1;
  double best = 1e300;
  int best_s = smin;
  for (int s = smin; s <= smax; ++s) {
    const int c = (chunks + s - 1) / s;
    if ((chunks + c - 1) / c != s) continue;   // would leave empty splits
    const int64_t waves = (static_cast<int64_t>(bh) * s + slots - 1) / slots;
    const double cost = static_cast<double>(waves) * (c + kCtaOverheadChunks) * (1.0 + 1e-3 * s);
    if (cost < best) {
      best = cost;
      best_s = s;
    }
  }
  *splits = best_s;
  *cps = (chunks + best_s - 1) / best_s;
}

struct WsLayout {
  uint64_t err, counters, partials, total;
};

WsLayout ws_layout(int64_t bh, int D, int32_t max_seq_len) {
  WsLayout w;
  w.err = 0;
  w.counters = kAlign;
  w.partials = align_up(w.counters + static_cast<uint64_t>(bh) * 4, kAlign);
  w.total = align_up(w.partials + static_cast<uint64_t>(bh) * max_splits_of(max_seq_len) *
                                      (D + 2) * 4,
                     kAlign);
  return w;
}

const unsigned char* side_base(const rq_cache* c, int layer, int kv) {
  const unsigned char* b = static_cast<const unsigned char*>(kv ? c->v_base : c->k_base);
  return b + static_cast<uint64_t>(layer) * c->layer_bytes;
}

Comp comp_of(const rq_cache* c, int layer, int kv, int r) {
  Comp k;
  k.base = const_cast<unsigned char*>(side_base(c, layer, kv)) + c->comp_off[r];
  k.rec_bytes = c->rec_bytes[r];
  k.bits = c->layout.bits[r];
  k.group = c->layout.group[r];
  k.has_alpha = (r != anchor_of(&c->layout)) ? 1 : 0;
  k.meta16 = (c->layout.flags & RQ_FLAG_META16) ? 1 : 0;
  const float* means = kv ? c->v_means : c->k_means;
  const rq_layout& l = c->layout;
  k.mean = (means != nullptr && k.has_alpha)
               ? means + (static_cast<int64_t>(layer) * l.num_loops + r) * l.kv_heads * l.head_dim
               : nullptr;
  k.heads = l.kv_heads;
  return k;
}

// Reference chain used to reconstruct loop `loop`: [loop, ..., anchor]
// (shared anchor: [loop, anchor]; the anchor loop alone is [anchor]).
int chain_of(const rq_cache* c, int layer, int kv, int loop, Comp* out) {
  const rq_layout* l = &c->layout;
  const int a = anchor_of(l);
  int n = 0;
  int r = loop;
  out[n++] = comp_of(c, layer, kv, r);
  while (r != a) {
    r = reference_of(l, r);
    out[n++] = comp_of(c, layer, kv, r);
  }
  return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Dense rotation of (layer, side) or nullptr (Hadamard).
const uint16_t* rot_of(const rq_cache* c, int layer, int kv) {
  const void* r = kv ? c->v_rot : c->k_rot;
  if (r == nullptr) return nullptr;
  const rq_layout& l = c->layout;
  return static_cast<const uint16_t*>(r) +
         static_cast<int64_t>(layer) * l.kv_heads * l.head_dim * l.head_dim;
}

rq_status check_cache(const rq_cache* c, int32_t layer, int32_t kv) {
  if (c == nullptr || c->k_base == nullptr || c->v_base == nullptr) return RQ_ERR_INVALID_ARG;
  if (rq_layout_validate(&c->layout) != RQ_OK) return RQ_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->layout.num_layers) return RQ_ERR_INVALID_ARG;
  if (kv != 0 && kv != 1) return RQ_ERR_INVALID_ARG;
  return RQ_OK;
}

rq_status check_range(const rq_cache* c, int32_t t0, int32_t n) {
  if (t0 < 0 || n < 0) return RQ_ERR_INVALID_ARG;
  if (static_cast<int64_t>(t0) + n > c->layout.max_tokens) return RQ_ERR_CAPACITY;
  return RQ_OK;
}

float rot_scale_of(int D) { return static_cast<float>(1.0 / sqrt(static_cast<double>(D))); }

float scale_log2_of(float softmax_scale, int D) {
  const double s = softmax_scale == 0.0f ? 1.0 / sqrt(static_cast<double>(D)) : softmax_scale;
  return static_cast<float>(s * 1.4426950408889634);
}

}  // namespace

extern "C" {

int32_t rq_abi_version(void) { return RQ_ABI_VERSION; }

const char* rq_status_string(rq_status s) {
  switch (s) {
    case RQ_OK: return "RQ_OK";
    case RQ_ERR_INVALID_ARG: return "RQ_ERR_INVALID_ARG";
    case RQ_ERR_UNSUPPORTED: return "RQ_ERR_UNSUPPORTED";
    case RQ_ERR_CAPACITY: return "RQ_ERR_CAPACITY";
    case RQ_ERR_CUDA: return "RQ_ERR_CUDA";
    case RQ_ERR_TIMEOUT: return "RQ_ERR_TIMEOUT";
    case RQ_ERR_WORKSPACE: return "RQ_ERR_WORKSPACE";
  }
  return "RQ_ERR_UNKNOWN";
}

rq_status rq_layout_validate(const rq_layout* l) {
  if (l == nullptr) return RQ_ERR_INVALID_ARG;
  if (l->num_layers < 1 || l->num_loops < 1 || l->num_loops > RQ_MAX_LOOPS) return RQ_ERR_INVALID_ARG;
  if (l->batch < 1 || l->kv_heads < 1 || l->max_tokens < 1) return RQ_ERR_INVALID_ARG;
  if (l->policy < RQ_POLICY_LAST_LOOP || l->policy > RQ_POLICY_PREVIOUS_LOOP)
    return RQ_ERR_INVALID_ARG;
  if ((l->flags & ~(RQ_FLAG_UNIT_ALPHA | RQ_FLAG_META16)) != 0) return RQ_ERR_INVALID_ARG;
  if (!is_pow2(l->head_dim) || l->head_dim < 32 || l->head_dim > 256) return RQ_ERR_INVALID_ARG;
  if (l->head_dim != 64 && l->head_dim != 128) return RQ_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(l->batch) * l->kv_heads > 65535) return RQ_ERR_UNSUPPORTED;
  if (l->max_tokens > (1 << 30)) return RQ_ERR_UNSUPPORTED;
  for (int r = 0; r < l->num_loops; ++r) {
    const int b = l->bits[r], g = l->group[r];
    if (b != 2 && b != 4) return RQ_ERR_INVALID_ARG;
    if (!is_pow2(g) || g < 16 || g > 128 || g > l->head_dim) return RQ_ERR_INVALID_ARG;
    if (g * b < 32) return RQ_ERR_INVALID_ARG;
  }
  return RQ_OK;
}

uint64_t rq_layer_bytes(const rq_layout* l) {
  if (rq_layout_validate(l) != RQ_OK) return 0;
  uint64_t c[RQ_MAX_LOOPS];
  uint32_t rb[RQ_MAX_LOOPS];
  return layout_offsets(l, c, rb);
}

uint64_t rq_cache_bytes(const rq_layout* l) {
  const uint64_t lb = rq_layer_bytes(l);
  return lb * (lb ? static_cast<uint64_t>(l->num_layers) : 0);
}

rq_status rq_cache_bind(const rq_layout* l, void* k_base, void* v_base, rq_cache* out) {
  if (out == nullptr || k_base == nullptr || v_base == nullptr) return RQ_ERR_INVALID_ARG;
  const rq_status st = rq_layout_validate(l);
  if (st != RQ_OK) return st;
  if (!aligned(k_base, kAlign) || !aligned(v_base, kAlign)) return RQ_ERR_INVALID_ARG;
  memset(out, 0, sizeof(*out));
  out->layout = *l;
  out->k_base = k_base;
  out->v_base = v_base;
  out->layer_bytes = layout_offsets(l, out->comp_off, out->rec_bytes);
  out->token_stride = token_stride_of(l);
  return RQ_OK;
}

rq_status rq_cache_set_means(rq_cache* c, const float* k_means, const float* v_means) {
  if (c == nullptr) return RQ_ERR_INVALID_ARG;
  if ((k_means != nullptr && !aligned(k_means, 16)) || (v_means != nullptr && !aligned(v_means, 16)))
    return RQ_ERR_INVALID_ARG;
  c->k_means = k_means;
  c->v_means = v_means;
  return RQ_OK;
}

rq_status rq_cache_set_rotations(rq_cache* c, const void* k_rot, const void* v_rot) {
  if (c == nullptr) return RQ_ERR_INVALID_ARG;
  if ((k_rot != nullptr && !aligned(k_rot, 16)) || (v_rot != nullptr && !aligned(v_rot, 16)))
    return RQ_ERR_INVALID_ARG;
  if ((k_rot != nullptr || v_rot != nullptr) && c->layout.head_dim != 128)
    return RQ_ERR_UNSUPPORTED;
  c->k_rot = k_rot;
  c->v_rot = v_rot;
  return RQ_OK;
}

rq_status rq_quantize_anchor(const rq_cache* c, int32_t layer, int32_t kv, const void* x,
                             int32_t t0, int32_t n, void* stream) {
  rq_status st = check_cache(c, layer, kv);
  if (st != RQ_OK) return st;
  if ((st = check_range(c, t0, n)) != RQ_OK) return st;
  if (n == 0) return RQ_OK;
  if (x == nullptr || !aligned(x, 16)) return RQ_ERR_INVALID_ARG;
  const rq_layout& l = c->layout;
  const int a = anchor_of(&l);
  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.x = static_cast<const uint16_t*>(x);
  p.bh = l.batch * l.kv_heads;
  p.n = n;
  p.t0 = t0;
  p.nblk = c->token_stride / kBlock;
  p.dst = comp_of(c, layer, kv, a);
  p.nref = 0;
  p.rot_scale = rot_scale_of(l.head_dim);
  p.urot = rot_of(c, layer, kv);
  p.heads = l.kv_heads;
  return cuda_status(launch_quantize(p, l.head_dim, l.bits[a], l.group[a], as_stream(stream)));
}

rq_status rq_quantize_append_residual(const rq_cache* c, int32_t layer, int32_t kv, int32_t loop,
                                      const void* x, int32_t t0, int32_t n, void* stream) {
  rq_status st = check_cache(c, layer, kv);
  if (st != RQ_OK) return st;
  const rq_layout& l = c->layout;
  if (loop < 0 || loop >= l.num_loops || loop == anchor_of(&l)) return RQ_ERR_INVALID_ARG;
  if ((st = check_range(c, t0, n)) != RQ_OK) return st;
  if (n == 0) return RQ_OK;
  if (x == nullptr || !aligned(x, 16)) return RQ_ERR_INVALID_ARG;
  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.x = static_cast<const uint16_t*>(x);
  p.bh = l.batch * l.kv_heads;
  p.n = n;
  p.t0 = t0;
  p.nblk = c->token_stride / kBlock;
  p.dst = comp_of(c, layer, kv, loop);
  // Reference: the anchor (shared policies) or the chain toward it.
  Comp chain[RQ_MAX_LOOPS];
  const int len = chain_of(c, layer, kv, loop, chain);   // [loop, ref...]
  p.nref = len - 1;
  for (int i = 1; i < len; ++i) p.ref[i - 1] = chain[i];
  p.unit_alpha = (l.flags & RQ_FLAG_UNIT_ALPHA) ? 1 : 0;
  p.rot_scale = rot_scale_of(l.head_dim);
  p.urot = rot_of(c, layer, kv);
  p.heads = l.kv_heads;
  return cuda_status(
      launch_quantize(p, l.head_dim, l.bits[loop], l.group[loop], as_stream(stream)));
}

rq_status rq_quantize_append_loops(const rq_cache* c, int32_t layer, const void* xk,
                                   const void* xv, int32_t t0, int32_t n, void* stream) {
  rq_status st = check_cache(c, layer, 0);
  if (st != RQ_OK) return st;
  if ((st = check_range(c, t0, n)) != RQ_OK) return st;
  if (xk == nullptr && xv == nullptr) return RQ_ERR_INVALID_ARG;
  if ((xk != nullptr && !aligned(xk, 16)) || (xv != nullptr && !aligned(xv, 16)))
    return RQ_ERR_INVALID_ARG;
  if (n == 0) return RQ_OK;
  const rq_layout& l = c->layout;
  QuantLoopsParams p;
  memset(&p, 0, sizeof(p));
  p.x[0] = static_cast<const uint16_t*>(xk);
  p.x[1] = static_cast<const uint16_t*>(xv);
  p.bh = l.batch * l.kv_heads;
  p.n = n;
  p.nloops = l.num_loops;
  p.anchor = anchor_of(&l);
  p.chained = chained_of(&l) ? 1 : 0;
  p.unit_alpha = (l.flags & RQ_FLAG_UNIT_ALPHA) ? 1 : 0;
  // residual loops away from the anchor, so every reference is stored first
  for (int k = 0, r = 0; r < l.num_loops; ++r) {
    const int rr = p.anchor == 0 ? r : l.num_loops - 1 - r;
    if (rr != p.anchor) p.order[k++] = rr;
  }
  p.t0 = t0;
  p.nblk = c->token_stride / kBlock;
  for (int kv = 0; kv < 2; ++kv)
    for (int r = 0; r < l.num_loops; ++r) p.dst[kv][r] = comp_of(c, layer, kv, r);
  p.rot_scale = rot_scale_of(l.head_dim);
  p.urot[0] = rot_of(c, layer, 0);
  p.urot[1] = rot_of(c, layer, 1);
  p.heads = l.kv_heads;
  return cuda_status(launch_quantize_loops(p, l.head_dim, as_stream(stream)));
}

rq_status rq_dequantize(const rq_cache* c, int32_t layer, int32_t kv, int32_t loop, int32_t t0,
                        int32_t n, float* out, void* stream) {
  rq_status st = check_cache(c, layer, kv);
  if (st != RQ_OK) return st;
  const rq_layout& l = c->layout;
  if (loop < 0 || loop >= l.num_loops) return RQ_ERR_INVALID_ARG;
  if ((st = check_range(c, t0, n)) != RQ_OK) return st;
  if (n == 0) return RQ_OK;
  if (out == nullptr || !aligned(out, 16)) return RQ_ERR_INVALID_ARG;
  DequantParams p;
  memset(&p, 0, sizeof(p));
  p.bh = l.batch * l.kv_heads;
  p.n = n;
  p.t0 = t0;
  p.nblk = c->token_stride / kBlock;
  p.ncomp = chain_of(c, layer, kv, loop, p.comp);
  p.rot_scale = rot_scale_of(l.head_dim);
  p.out = out;
  p.urot = rot_of(c, layer, kv);
  p.heads = l.kv_heads;
  return cuda_status(launch_dequantize(p, l.head_dim, as_stream(stream)));
}

uint64_t rq_decode_workspace_bytes(const rq_layout* l, int32_t max_seq_len) {
  if (rq_layout_validate(l) != RQ_OK || max_seq_len < 0) return 0;
  return ws_layout(static_cast<int64_t>(l->batch) * l->kv_heads, l->head_dim, max_seq_len).total;
}

uint64_t rq_decode_bf16_workspace_bytes(int32_t batch, int32_t heads, int32_t head_dim,
                                        int32_t max_seq_len) {
  if (batch < 1 || heads < 1 || (head_dim != 64 && head_dim != 128) || max_seq_len < 0) return 0;
  return ws_layout(static_cast<int64_t>(batch) * heads, head_dim, max_seq_len).total;
}

rq_status rq_decode_workspace_init(void* ws, uint64_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes == 0) return RQ_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, as_stream(stream)));
}

rq_status rq_workspace_error(void* ws, uint64_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < 4) return RQ_ERR_INVALID_ARG;
  uint32_t h = 0;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(&h, ws, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && h != 0) {
    e = cudaMemsetAsync(ws, 0, 4, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return RQ_ERR_CUDA;
  if (h & kErrTimeout) return RQ_ERR_TIMEOUT;
  if (h & kErrRange) return RQ_ERR_UNSUPPORTED;
  if (h & kErrSeqLen) return RQ_ERR_CAPACITY;
  return RQ_OK;
}

static rq_status fill_decode_params(const rq_cache* c, int32_t layer, int32_t loop,
                                    int32_t max_seq_len, DecodeParams* p, int* D) {
  const rq_layout& l = c->layout;
  memset(p, 0, sizeof(*p));
  p->bh = l.batch * l.kv_heads;
  p->heads = l.kv_heads;
  p->nblk = c->token_stride / kBlock;
  p->ncomp = chain_of(c, layer, 0, loop, p->k);
  (void)chain_of(c, layer, 1, loop, p->v);
  p->max_seq_len = max_seq_len;
  p->rot_scale = rot_scale_of(l.head_dim);
  p->urot_k = rot_of(c, layer, 0);
  p->urot_v = rot_of(c, layer, 1);
  *D = l.head_dim;
  int stages = 0, occ = 0, chunk = kChunk;
  if (fast_decode_plan(*p, *D, &stages, &chunk, &occ)) {
    p->use_fast = 1;
  } else {
    chunk = kChunk;
    p->use_fast = 0;
    p->stage_bytes = decode_stage_bytes(*p, *D);
    stages = static_cast<int>(kRingBudget / p->stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 1 && 2 * kRingBudget >= p->stage_bytes) stages = 1;
    if (stages < 1) return RQ_ERR_UNSUPPORTED;
    if (decode_occupancy(*D, decode_dyn_smem(*D, stages, p->stage_bytes), &occ) != cudaSuccess)
      return RQ_ERR_CUDA;
  }
  p->stages = stages;
  p->chunk = chunk;
  choose_splits(p->bh, max_seq_len, chunk, occ, &p->splits, &p->chunks_per_split);
  return RQ_OK;
}

rq_status rq_selftest_wait_timeout(void* workspace, uint64_t ws_bytes, int32_t limit_ms,
                                   void* stream) {
  if (workspace == nullptr || !aligned(workspace, kAlign) || ws_bytes < kAlign)
    return RQ_ERR_INVALID_ARG;
  if (limit_ms < 1 || limit_ms > 1000) return RQ_ERR_INVALID_ARG;
  uint32_t* err = static_cast<uint32_t*>(workspace);   // the error word (offset 0)
  return cuda_status(launch_selftest_wait(err, static_cast<uint64_t>(limit_ms) * 1000000ull,
                                          as_stream(stream)));
}

int32_t rq_decode_splits(const rq_layout* l, int32_t max_seq_len) {
  if (rq_layout_validate(l) != RQ_OK || max_seq_len < 0) return 0;
  // Shape-only: a cache bound to dummy (aligned, never dereferenced) bases.
  rq_cache c;
  if (rq_cache_bind(l, reinterpret_cast<void*>(kAlign), reinterpret_cast<void*>(kAlign), &c) !=
      RQ_OK)
    return 0;
  DecodeParams p;
  int D = 0;
  // the loop farthest from the anchor is the most expensive to decode
  const int far = anchor_of(l) == 0 ? l->num_loops - 1 : 0;
  if (fill_decode_params(&c, 0, far, max_seq_len, &p, &D) != RQ_OK) return 0;
  return p.splits;
}

rq_status rq_plan_splits(int32_t rows, int32_t max_seq_len, int32_t ctas_per_sm, int32_t sms,
                         int32_t* splits, int32_t* chunks_per_split) {
  if (rows < 1 || max_seq_len < 0 || ctas_per_sm < 1 || sms < 1 || splits == nullptr ||
      chunks_per_split == nullptr)
    return RQ_ERR_INVALID_ARG;
  int s = 0, c = 0;
  choose_splits_on(rows, max_seq_len, kChunk, ctas_per_sm, sms, &s, &c);
  *splits = s;
  *chunks_per_split = c;
  return RQ_OK;
}

rq_status rq_decode_attention(const rq_cache* c, int32_t layer, int32_t loop, const void* q,
                              const int32_t* seq_lens, int32_t max_seq_len, const void* k_cur,
                              const void* v_cur, float softmax_scale, float* out,
                              void* workspace, uint64_t ws_bytes, void* stream) {
  rq_status st = check_cache(c, layer, 0);
  if (st != RQ_OK) return st;
  const rq_layout& l = c->layout;
  if (loop < 0 || loop >= l.num_loops) return RQ_ERR_INVALID_ARG;
  if (q == nullptr || seq_lens == nullptr || k_cur == nullptr || v_cur == nullptr ||
      out == nullptr || workspace == nullptr)
    return RQ_ERR_INVALID_ARG;
  if (max_seq_len < 0) return RQ_ERR_INVALID_ARG;
  if (max_seq_len > l.max_tokens) return RQ_ERR_CAPACITY;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return RQ_ERR_INVALID_ARG;
  if (!aligned(workspace, kAlign)) return RQ_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(static_cast<int64_t>(l.batch) * l.kv_heads, l.head_dim, max_seq_len);
  if (ws_bytes < w.total) return RQ_ERR_WORKSPACE;
  DecodeParams p;
  int D = 0;
  if ((st = fill_decode_params(c, layer, loop, max_seq_len, &p, &D)) != RQ_OK) return st;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.q = static_cast<const uint16_t*>(q);
  p.kcur = static_cast<const uint16_t*>(k_cur);
  p.vcur = static_cast<const uint16_t*>(v_cur);
  p.seq_lens = seq_lens;
  p.scale_log2 = scale_log2_of(softmax_scale, D);
  p.out = out;
  p.err = reinterpret_cast<uint32_t*>(ws + w.err);
  p.counters = reinterpret_cast<uint32_t*>(ws + w.counters);
  p.partials = reinterpret_cast<float*>(ws + w.partials);
  return cuda_status(p.use_fast ? launch_decode_fast(p, D, as_stream(stream))
                                : launch_decode(p, D, as_stream(stream)));
}

rq_status rq_decode_attention_bf16(int32_t batch, int32_t heads, int32_t head_dim, const void* q,
                                   const void* k, const void* v, int64_t token_stride,
                                   const int32_t* seq_lens, int32_t max_seq_len,
                                   const void* k_cur, const void* v_cur, float softmax_scale,
                                   float* out, void* workspace, uint64_t ws_bytes,
                                   void* stream) {
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > 65535)
    return RQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return RQ_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || seq_lens == nullptr || k_cur == nullptr ||
      v_cur == nullptr || out == nullptr || workspace == nullptr)
    return RQ_ERR_INVALID_ARG;
  if (max_seq_len < 0 || token_stride < max_seq_len || token_stride < 1) return RQ_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(workspace, kAlign))
    return RQ_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return RQ_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(static_cast<int64_t>(batch) * heads, head_dim, max_seq_len);
  if (ws_bytes < w.total) return RQ_ERR_WORKSPACE;
  DecodeBf16Params p;
  memset(&p, 0, sizeof(p));
  p.bh = batch * heads;
  p.heads = heads;
  p.tstride = token_stride;
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.q = static_cast<const uint16_t*>(q);
  p.kcur = static_cast<const uint16_t*>(k_cur);
  p.vcur = static_cast<const uint16_t*>(v_cur);
  p.seq_lens = seq_lens;
  p.max_seq_len = max_seq_len;
  p.scale_log2 = scale_log2_of(softmax_scale, head_dim);
  p.out = out;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.err = reinterpret_cast<uint32_t*>(ws + w.err);
  p.counters = reinterpret_cast<uint32_t*>(ws + w.counters);
  p.partials = reinterpret_cast<float*>(ws + w.partials);
  p.stage_bytes = bf16_stage_bytes(head_dim);
  int stages = static_cast<int>(kRingBudget / p.stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) stages = 2;
  p.stages = stages;
  int occ = 0;
  if (bf16_occupancy(head_dim, stages, &occ) != cudaSuccess) return RQ_ERR_CUDA;
  choose_splits(p.bh, max_seq_len, bf16_chunk(head_dim), occ, &p.splits, &p.chunks_per_split);
  return cuda_status(launch_decode_bf16(p, head_dim, as_stream(stream)));
}

}  // extern "C"

namespace rq {
rq_status plan_decode(const rq_cache* c, int32_t layer, int32_t loop, int32_t max_seq_len,
                      DecodeParams* p, int* D) {
  return fill_decode_params(c, layer, loop, max_seq_len, p, D);
}
float decode_scale_log2(float softmax_scale, int D) { return scale_log2_of(softmax_scale, D); }
}  // namespace rq
