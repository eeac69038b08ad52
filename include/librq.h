/*
 * librq.h -- C ABI of librq, a B200-native (sm_100a) implementation of the
 * ResidualQuant KV-cache hot path for looped Transformers.
 *
 * Citations: [RQ §x] = "ResidualQuant: KV Cache Quantization for Looped
 * Transformers with 2-Bit Residuals" (paperpeel.com/paper/2610.10381).
 *
 * What is stored [RQ §3.2, §3.3, §3.4, App. D, App. G.2]:
 *   For every past token and KV head of loop r, with Z = H x the normalised
 *   Sylvester-Hadamard rotation of the bf16 row x:
 *     anchor loop a:            A = deq(Q_ba(Z_a))
 *     every other loop r:       alpha_r = <Z_r, R>/<R, R> (1 with
 *                               RQ_FLAG_UNIT_ALPHA), alpha~ = bf16(alpha_r),
 *                               codes of Q_br(Z_r - alpha~ R)
 *   where the policy fixes a and R [RQ §3.2 reference KV, §5.2]:
 *     RQ_POLICY_LAST_LOOP      a = L-1, R = A (shared final-loop anchor)
 *     RQ_POLICY_NEXT_LOOP      a = L-1, R = Z^_{r+1} (chain toward the anchor)
 *     RQ_POLICY_FIRST_LOOP     a = 0,   R = A (shared first-loop anchor)
 *     RQ_POLICY_PREVIOUS_LOOP  a = 0,   R = Z^_{r-1} (chain toward the anchor)
 *   Q_b is group-wise affine quantisation [RQ §2.1]: per group of g
 *   consecutive channels, s = (max - min)/(2^b - 1), s~ = fp16(s),
 *   z~ = fp16(min), code = rint_even(clamp((z - z~) * (1/s~), 0, 2^b - 1)).
 *   Reconstruction: Z^_r = alpha~_r R + s~ c + z~ and X^_r = H^T Z^_r.
 *   With fixed means (rq_cache_set_means) a residual loop stores the codes
 *   of Z_r - mu_r - alpha~ R and adds mu_r back; with dense rotations
 *   (rq_cache_set_rotations) Z = U x replaces H x and X^ = U^T Z^.
 *
 * Storage contract (per layer and per side K | V):
 *   Tokens are stored in records of RQ_BLOCK_TOKENS = 32 consecutive tokens.
 *   Loop r of (row = batch*kv_heads index b*H + h, block k) is one record at
 *   byte offset comp_off[r] + (row * token_stride/32 + k) * rec_bytes[r] of
 *   the (layer, side) region; token_stride is max_tokens rounded up to 64
 *   (an even number of records per row).
 *   A record holds, contiguously:
 *     codes  uint32 [32][head_dim * bits[r] / 32]
 *     meta   uint32 [32][head_dim / group[r]]; low half fp16 scale s~,
 *            high half fp16 offset z~ (with RQ_FLAG_META16: uint16
 *            [32][head_dim / group[r]], scale byte | offset byte << 8, where
 *            s~ = (1 + m/8) 2^(E - 18) for the byte 8E + m, E = 0 meaning 0;
 *            s~ is the nearest such value to max((max - min)/(2^b - 1),
 *            |min|/15.875) (below the range: the smallest; above: the
 *            largest) and zq = clamp(floor(8 min / s~), -128, 127))
 *     alpha  bf16   [32]             (residual loops only)
 *   so a decode stage of one component (one or two records) is one
 *   contiguous copy.
 *   Code order inside a token's row: b = 2: channel i in word i/16, bits
 *   [2*(i%16), +2).  b = 4: in blocks of 16 channels, i = 16u + v, word
 *   2u + ((v>>1)&1), bits [4*(2*(v>>2) + (v&1)), +4).  Little-endian words.
 *   Effective bits per element of loop r: bits[r] + 32/group[r] (16/group[r]
 *   with RQ_FLAG_META16)
 *   (+ 16/head_dim for a residual loop).  Components are laid out anchor
 *   first, then the other loops in increasing index (comp_off).
 *
 * Conventions for every entry point:
 *   - All pointers except rq_layout / rq_cache arguments are DEVICE pointers
 *     unless stated; the caller owns all memory.  librq allocates nothing,
 *     keeps no per-call state, and is safe to call from several host threads
 *     on different streams.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on that stream.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns an error and launches nothing.  Launch failures return
 *     RQ_ERR_CUDA.  Device code never traps; conditions only the device can
 *     see (a sequence length over its bound, a bounded wait that ran out) are
 *     recorded in the decode workspace and reported by rq_workspace_error().
 *   - bf16 / fp16 tensors are passed as raw 16-bit words.
 */
#ifndef LIBRQ_H
#define LIBRQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RQ_ABI_VERSION 3
#define RQ_MAX_LOOPS 32
#define RQ_BLOCK_TOKENS 32

typedef enum rq_status {
  RQ_OK = 0,
  RQ_ERR_INVALID_ARG = 1,   /* null pointer, bad index, misaligned buffer ... */
  RQ_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. head_dim 96)        */
  RQ_ERR_CAPACITY = 3,      /* token range or sequence length over capacity  */
  RQ_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
  RQ_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out             */
  RQ_ERR_WORKSPACE = 6      /* workspace too small                            */
} rq_status;

/* Reference policy [RQ §3.2, §5.2, App. D]. */
typedef enum rq_policy {
  RQ_POLICY_LAST_LOOP = 0,     /* anchor L-1; every loop references the anchor  */
  RQ_POLICY_NEXT_LOOP = 1,     /* anchor L-1; loop r references loop r+1        */
  RQ_POLICY_FIRST_LOOP = 2,    /* anchor 0; every loop references the anchor    */
  RQ_POLICY_PREVIOUS_LOOP = 3  /* anchor 0; loop r references loop r-1          */
} rq_policy;

/* rq_layout.flags */
#define RQ_FLAG_UNIT_ALPHA 1   /* alpha_r = 1: plain differences, no LS scaling
                                  [RQ §3.1-§3.2, Table 3 "w/o LS scaling"] */
#define RQ_FLAG_META16 2       /* 16 bits of metadata per group [RQ §5.1,
                                  App. A.3]: meta uint16 = scale byte (unsigned
                                  e5m3, bias 18, 0 = zero scale) | offset byte
                                  (int8 zq, z~ = zq * s~ / 8) << 8; see below */

/* Shape and precision of a compressed KV cache.
 *   num_layers  >= 1
 *   num_loops   L in [1, RQ_MAX_LOOPS]; the anchor is loop L-1 (Last-/Next-
 *               loop) or loop 0 (First-/Previous-loop)
 *   batch, kv_heads >= 1
 *   head_dim    D in {64, 128}
 *   max_tokens  token capacity per (batch, head), >= 1
 *   policy      rq_policy
 *   flags       0 or RQ_FLAG_UNIT_ALPHA | RQ_FLAG_META16
 *   bits[r]     2 or 4
 *   group[r]    g in {16, 32, 64, 128}, g divides D, g * bits[r] >= 32
 */
typedef struct rq_layout {
  int32_t num_layers;
  int32_t num_loops;
  int32_t batch;
  int32_t kv_heads;
  int32_t head_dim;
  int32_t max_tokens;
  int32_t policy;
  int32_t flags;               /* RQ_FLAG_* */
  int32_t bits[RQ_MAX_LOOPS];
  int32_t group[RQ_MAX_LOOPS];
} rq_layout;

/* A cache bound to caller-owned device memory (filled by rq_cache_bind;
 * treat as read-only).  Offsets are bytes within one (layer, side). */
typedef struct rq_cache {
  rq_layout layout;
  void* k_base;                      /* num_layers * layer_bytes, K side */
  void* v_base;                      /* num_layers * layer_bytes, V side */
  uint64_t layer_bytes;
  int64_t token_stride;              /* max_tokens rounded up to 64 */
  uint64_t comp_off[RQ_MAX_LOOPS];   /* first record of loop r (256-B aligned) */
  uint32_t rec_bytes[RQ_MAX_LOOPS];  /* bytes of one 32-token record of loop r */
  const float* k_means;              /* fixed means (rq_cache_set_means) or NULL */
  const float* v_means;
  const void* k_rot;                 /* dense rotations (rq_cache_set_rotations) or NULL */
  const void* v_rot;
} rq_cache;

/* ABI version of the loaded library (RQ_ABI_VERSION at build time). */
int32_t rq_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* rq_status_string(rq_status s);

/* Checks every field of a layout.  RQ_OK, RQ_ERR_INVALID_ARG or
 * RQ_ERR_UNSUPPORTED (head_dim or a bit width this build does not have). */
rq_status rq_layout_validate(const rq_layout* layout);

/* Bytes of ONE side (K or V) for all layers; 0 if the layout is invalid.
 * The caller allocates this much twice (K and V). */
uint64_t rq_cache_bytes(const rq_layout* layout);

/* Bytes of one (layer, side): the stride between layers inside a side. */
uint64_t rq_layer_bytes(const rq_layout* layout);

/* Fixed means of the residual loops [RQ App. G.2]: the reconstruction of a
 * residual loop r is Z^_r = alpha~_r R + D(c_r) + mu_r, and the encoder
 * removes mu_r before the LS coefficient (zc = Z_r - mu_r, alpha =
 * <zc, R>/<R, R>, codes of zc - alpha~ R).  k_means, v_means: device fp32
 * [num_layers][num_loops][kv_heads][head_dim] in the rotated domain (the
 * anchor loop's rows are not read), 16-byte aligned, or NULL for no means
 * (the state after rq_cache_bind).  The cache keeps the pointers; the caller
 * keeps the buffers alive and unchanged while appends and decodes that use
 * them are in flight.  Appends and decodes of one cache must see the same
 * means. */
rq_status rq_cache_set_means(rq_cache* cache, const float* k_means, const float* v_means);

/* Dense rotations in place of the Sylvester-Hadamard transform [RQ §3.3,
 * App. G.1, App. G.2]: one matrix per (layer, head) and side, shared by every
 * loop, stored in binary16; the quantisers compute Z = U x with x rounded
 * from bf16 to binary16 and fp32 accumulation on the tensor cores, decode
 * scores use U_K q (q rounded to binary16, fp32 accumulation) and the output
 * is U_V^T of the fp32 value sum; rq_dequantize returns U^T Z^.
 *   k_rot, v_rot  device binary16 [num_layers][kv_heads][head_dim][head_dim],
 *                 row i of a matrix giving output channel i (z_i = sum_j
 *                 U_ij x_j), 16-byte aligned; NULL for a side keeps the
 *                 Hadamard transform (the state after rq_cache_bind).
 * head_dim must be 128 when either is set (RQ_ERR_UNSUPPORTED otherwise).
 * The cache keeps the pointers; the caller keeps the matrices alive and
 * unchanged while appends and decodes that use them are in flight.  The
 * accumulation order of a tensor-core product is the hardware's, so the
 * codes are those of some fp32 ordering of the exact binary16 products (the
 * pages fix the formats, not the order). */
rq_status rq_cache_set_rotations(rq_cache* cache, const void* k_rot, const void* v_rot);

/* Binds device buffers of rq_cache_bytes() each (256-byte aligned) to `out`.
 * The buffers need no initialisation.  Host-only, launches nothing. */
rq_status rq_cache_bind(const rq_layout* layout, void* k_base, void* v_base,
                        rq_cache* out);

/* Quantise-and-append the anchor loop a (L-1, or 0 under First-/Previous-
 * loop) [RQ §3.2, §3.4, §4.2 Prefill / Decode]: rows x (bf16,
 * [batch][kv_heads][n][head_dim], contiguous) of loop a are rotated,
 * affine-quantised with bits[a] / group[a] and stored at token positions
 * [t0, t0 + n) of `layer`, side kv (0 = K, 1 = V).
 * n = 0 is a no-op.  t0 + n > max_tokens -> RQ_ERR_CAPACITY. */
rq_status rq_quantize_anchor(const rq_cache* cache, int32_t layer, int32_t kv,
                             const void* x, int32_t t0, int32_t n,
                             void* stream);

/* Quantise-and-append residual loop `loop` (any loop but the anchor) [RQ
 * §3.2 scaling coefficient, §3.3, App. G.1]: alpha, residual, rotation,
 * affine quantisation and bit-packing of rows x (same layout as above).
 * Stream-ordered precondition: the reference rows [t0, t0 + n) are stored
 * already -- the anchor (LAST_LOOP, FIRST_LOOP), loops loop+1 .. L-1
 * (NEXT_LOOP) or loops 0 .. loop-1 (PREVIOUS_LOOP). */
rq_status rq_quantize_append_residual(const rq_cache* cache, int32_t layer,
                                      int32_t kv, int32_t loop, const void* x,
                                      int32_t t0, int32_t n, void* stream);

/* Quantise-and-append of every loop of `layer` at token positions
 * [t0, t0 + n), K and V, in one launch [RQ §3.2, §3.4, §4.2 Decode: the new
 * token's loops are stored after the final loop]: the anchor and every other
 * loop against its reference (the anchor, or the chain Z^_{r+1} / Z^_{r-1}
 * processed away from the anchor).  Stores exactly the bytes of
 * rq_quantize_anchor followed by rq_quantize_append_residual for each loop in
 * the policy's order; the anchor is not re-read from the cache.
 *   xk, xv  bf16 [num_loops][batch][kv_heads][n][head_dim], contiguous,
 *           16-byte aligned; either may be NULL to skip that side (not both).
 * n = 0 is a no-op.  t0 + n > max_tokens -> RQ_ERR_CAPACITY. */
rq_status rq_quantize_append_loops(const rq_cache* cache, int32_t layer,
                                   const void* xk, const void* xv, int32_t t0,
                                   int32_t n, void* stream);

/* Reconstructs X^ of loop `loop` at positions [t0, t0 + n) in the original
 * (unrotated) domain into out (fp32, [batch][kv_heads][n][head_dim]).
 * For tests and export; not on the decode path [RQ App. G.2]. */
rq_status rq_dequantize(const rq_cache* cache, int32_t layer, int32_t kv,
                        int32_t loop, int32_t t0, int32_t n, float* out,
                        void* stream);

/* Workspace of rq_decode_attention for up to max_seq_len past tokens. */
uint64_t rq_decode_workspace_bytes(const rq_layout* layout,
                                   int32_t max_seq_len);

/* Zeroes a decode workspace (cudaMemsetAsync).  Required once after
 * allocation and after any call reported RQ_ERR_TIMEOUT; the kernels leave
 * the workspace ready for the next call otherwise. */
rq_status rq_decode_workspace_init(void* workspace, uint64_t ws_bytes,
                                   void* stream);

/* Compressed decode attention of loop `loop` for one query token per
 * (batch, head) [RQ §4.1, §4.2 Decode, App. G.2]:
 *   past keys/values t < seq_lens[b] are rebuilt on the fly from the packed
 *   cache (anchor + the loop's residual; the whole chain under NEXT_LOOP and
 *   PREVIOUS_LOOP),
 *   scores use the rotated query (Hq) . Z^_K, values are accumulated in the
 *   rotated domain and rotated back once; the current token's own k_cur /
 *   v_cur (bf16, unrotated, [batch][kv_heads][head_dim]) are merged with the
 *   softmax statistics.  Softmax and accumulation are fp32.
 *   q        bf16 [batch][kv_heads][head_dim]
 *   seq_lens int32 [batch] device array; values outside [0, max_seq_len] are
 *            clamped and flagged (rq_workspace_error -> RQ_ERR_CAPACITY)
 *   max_seq_len  host bound on seq_lens, <= max_tokens (sizes the grid)
 *   softmax_scale  0 selects 1/sqrt(head_dim)
 *   out      fp32 [batch][kv_heads][head_dim]; the row of a (batch, head)
 *            whose decode is not valid (a bounded wait ran out, or a value
 *            weight left the accumulator range, see rq_workspace_error) is
 *            written as NaN
 *   workspace  >= rq_decode_workspace_bytes(layout, max_seq_len), zeroed by
 *            rq_decode_workspace_init once; calls sharing a workspace must be
 *            ordered on one stream, and a workspace moved to a layout with
 *            another batch * kv_heads must be zeroed again (its per-row
 *            counters sit where the other layout's partials were). */
rq_status rq_decode_attention(const rq_cache* cache, int32_t layer,
                              int32_t loop, const void* q,
                              const int32_t* seq_lens, int32_t max_seq_len,
                              const void* k_cur, const void* v_cur,
                              float softmax_scale, float* out, void* workspace,
                              uint64_t ws_bytes, void* stream);

/* Uncompressed BF16 decode attention on the same split-K engine: the
 * baseline the compressed path is measured against.
 *   k, v  bf16 [batch][heads][token_stride][head_dim]
 *   other arguments as rq_decode_attention; head_dim in {64, 128}. */
uint64_t rq_decode_bf16_workspace_bytes(int32_t batch, int32_t heads,
                                        int32_t head_dim, int32_t max_seq_len);
rq_status rq_decode_attention_bf16(int32_t batch, int32_t heads,
                                   int32_t head_dim, const void* q,
                                   const void* k, const void* v,
                                   int64_t token_stride,
                                   const int32_t* seq_lens,
                                   int32_t max_seq_len, const void* k_cur,
                                   const void* v_cur, float softmax_scale,
                                   float* out, void* workspace,
                                   uint64_t ws_bytes, void* stream);

/* Reads and clears the device-side error word of a decode workspace
 * (synchronises `stream`).  RQ_OK, RQ_ERR_CAPACITY (a seq_lens entry was out
 * of range), RQ_ERR_UNSUPPORTED (a value weight p_t * kappa * s~ reached
 * 2^36, outside the range of the decode kernel's scaled accumulators; the
 * affected output rows are NaN) or RQ_ERR_TIMEOUT (a bounded wait ran out;
 * the affected output rows are NaN; re-initialise the workspace). */
rq_status rq_workspace_error(void* workspace, uint64_t ws_bytes, void* stream);

/* Self-test of the device-side failure path (for tests): one CTA waits on an
 * mbarrier phase that nothing completes, with a limit of limit_ms of device
 * time (1..1000), records the timeout in the workspace's error word and
 * returns; rq_workspace_error then reports RQ_ERR_TIMEOUT and the context
 * stays usable.  workspace as for rq_decode_attention. */
rq_status rq_selftest_wait_timeout(void* workspace, uint64_t ws_bytes, int32_t limit_ms,
                                   void* stream);

/* Number of split-K partitions rq_decode_attention uses for this shape on
 * the current device (for tests and benchmarks). */
int32_t rq_decode_splits(const rq_layout* layout, int32_t max_seq_len);

/* The split plan alone, for a device with `sms` multiprocessors running
 * `ctas_per_sm` decode CTAs each (host logic, no device access; tests):
 * `rows` = batch * kv_heads units, 64-token chunks.  *splits >= 1 partitions of
 * *chunks_per_split chunks each, none empty, at most one per chunk (and at most
 * the workspace's bound); the count fills every resident slot at least once
 * when the sequence is long enough and minimises (waves of resident CTAs) x
 * (chunks per CTA + a fixed per-CTA cost).  RQ_ERR_INVALID_ARG for rows,
 * ctas_per_sm or sms below 1, a negative length or NULL outputs. */
rq_status rq_plan_splits(int32_t rows, int32_t max_seq_len, int32_t ctas_per_sm, int32_t sms,
                         int32_t* splits, int32_t* chunks_per_split);

/* rq_decode_attention for callers that cannot allocate device memory -- code
 * embedded in a host framework that owns every allocation, or a serving loop
 * that may not call cudaMalloc -- and so cannot provide a workspace.  The
 * paper has no counterpart; this is an interface convenience.
 *   Arguments, layouts and results are those of rq_decode_attention, minus
 *   the workspace.  The split-K scratch is a fixed 8 MiB array inside this
 *   library that every GPU which loads the library holds until exit.  The
 *   call allocates nothing (no cudaMalloc / cudaFree).
 *   The first call on a device looks up that array's address and zeroes it
 *   (synchronously, with that device current): make that first call before
 *   any CUDA-graph stream capture.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents; calls that overlap on the GPU (other streams, other host
 *   threads) race on it and must be ordered by the caller.
 *   If the split partials of a shape do not fit, fewer splits are used; if
 *   one split per (batch, head) does not fit (batch * kv_heads * (head_dim+2)
 *   * 4 bytes above the 8 MiB less 256 KiB of per-row counters) the call
 *   returns RQ_ERR_WORKSPACE without launching.  With no workspace there is no error word for the caller to
 *   read: a (batch, head) whose decode is not valid (a bounded wait ran out,
 *   or a value weight left the accumulator range) gets a NaN output row, as
 *   in rq_decode_attention; a seq_lens entry out of range is clamped without
 *   a report. */
rq_status rq_decode_attention_noalloc(const rq_cache* cache, int32_t layer,
                                      int32_t loop, const void* q,
                                      const int32_t* seq_lens,
                                      int32_t max_seq_len, const void* k_cur,
                                      const void* v_cur, float softmax_scale,
                                      float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBRQ_H */
