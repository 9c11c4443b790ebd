/*
 * rq_api.h -- C ABI of the B200 ResidualQuant hot path (librq_b200.so).
 *
 * Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
 * 2-Bit Residuals" (Kim et al., 2026), cited below as [RQ].  A looped
 * Transformer writes one KV cache per loop.  The final loop's keys/values are
 * kept as the reference (bf16, or an INT4 "anchor"); every other loop l is
 * stored as a least-squares scaled, Hadamard-rotated, group-quantised residual
 *      K_l  ~  alpha_l * K_ref  +  H^T deq(codes_l)        (likewise V)
 * ([RQ] abstract; Figure 1 steps 2-5; Figure 2 caption).  Decode attention
 * scores each cached token as  alpha (q . K_ref) + (H q) . deq(codes)  and
 * never materialises a bf16 copy of loop l.  K_ref is the loop's anchor: the
 * final loop by default (see rq_anchor_policy).
 *
 * Conventions shared by every entry point:
 *  - Memory: the caller owns all device memory and streams.  The library
 *    allocates nothing on the device at run time; a cache handle holds only
 *    host metadata.  The one piece of device memory the library owns is a
 *    fixed RQ_STATIC_SCRATCH_BYTES array that every GPU loading the library
 *    holds until exit, used only by rq_decode_attention_static_scratch.
 *  - Asynchrony: calls that take a cudaStream_t enqueue work on that stream and
 *    return without synchronising (rq_get_error is the one exception).  The
 *    decode kernels are launched as programmatic dependents (CUDA's
 *    programmatic stream serialization): a decode kernel may be scheduled
 *    while the previous kernel on the stream finishes, but it touches no
 *    global memory before that kernel has completed, so stream order is kept;
 *    this also holds inside captured CUDA graphs.
 *  - Errors: argument errors are detected on the host before anything is
 *    enqueued and are returned as RQ_ERR_INVALID_ARG / RQ_ERR_UNSUPPORTED /
 *    RQ_ERR_CAPACITY / RQ_ERR_WORKSPACE; a failed launch returns RQ_ERR_CUDA.
 *    Conditions only the device can see (non-finite inputs, a length beyond
 *    capacity, a pipeline wait that timed out) set bits of the cache's device
 *    status word, read by rq_get_error.  rq_last_error_message() returns a
 *    human-readable reason for the calling thread's last non-OK status.
 *  - Devices: one process drives one device (one process per GPU).  Each decode
 *    kernel's shared-memory attribute is set once per process, on the device
 *    current at its first launch.
 *  - Loop index is 0-based; by default loop num_loops-1 is every loop's reference.
 *  - head_dim is 128 everywhere (the rotation is the order-128 Hadamard).
 *  - All tensors are row-major and contiguous unless strides are passed.
 */
#ifndef RQ_API_H
#define RQ_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of this header are the library's only exported names. */
#if defined(__GNUC__)
#define RQ_API __attribute__((visibility("default")))
#else
#define RQ_API
#endif

/* A CUDA stream handle (cudaStream_t); 0 is the legacy default stream. */
typedef void* rq_stream_t;

#define RQ_MAX_LOOPS 16
#define RQ_HEAD_DIM 128
/* Cache planes are laid out in pages of this many tokens: capacity is rounded
 * up to a multiple of it, and decode attention streams whole pages. */
#define RQ_PAGE_TOKENS 64
/* Largest batch a decode call accepts (per-sequence page offsets live in
 * shared memory). */
#define RQ_MAX_BATCH 1024

typedef enum rq_status {
  RQ_OK = 0,
  RQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size or misaligned buffer */
  RQ_ERR_UNSUPPORTED = 2,  /* a valid but unimplemented configuration */
  RQ_ERR_CAPACITY = 3,     /* tokens would land beyond the cache capacity */
  RQ_ERR_WORKSPACE = 4,    /* workspace smaller than *_workspace_size says */
  RQ_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
  RQ_ERR_DEVICE_FLAG = 6   /* rq_get_error: the device status word is set */
} rq_status;

/* Bits of the device status word (rq_get_error's *flags_out). */
#define RQ_FLAG_BAD_INPUT 1u      /* encode saw a non-finite value or |x| > 65504 */
#define RQ_FLAG_POSITION 2u       /* encode position + n_tokens beyond capacity (tokens dropped) */
#define RQ_FLAG_CTX_LEN 4u        /* decode ctx_len outside [0, capacity] (clamped) */
#define RQ_FLAG_PIPE_TIMEOUT 8u   /* a decode pipeline wait exceeded its limit (output invalid) */
#define RQ_FLAG_META_OVERFLOW 16u /* an alpha, scale or offset overflowed fp16 */

/* Scaling coefficient of the reference: [RQ] Figure 1 step 3 (least squares,
 * "LS"); Figure 3 caption ("alpha = 1" ablation); Figure 1 step 1 (direct
 * quantisation = alpha 0, no rotation); Table 9 ("Norm-ratio": ||x||/||ref||). */
typedef enum rq_alpha_mode {
  RQ_ALPHA_LS = 0,
  RQ_ALPHA_ONE = 1,
  RQ_ALPHA_ZERO = 2,
  RQ_ALPHA_NORM_RATIO = 3
} rq_alpha_mode;

/* Which loop is each loop's reference: [RQ] Table 1 ("First-loop",
 * "Last-loop" reference choice), Table 8 (anchor intervals N x [2^n, 4]:
 * groups of loops each ending in its own INT4 anchor) and Table 9 / Figure 3
 * caption (the "Previous-loop" and "Next-loop" reference family).
 * Under the two chained policies loop l is stored against the reconstruction
 *     x_hat_ref = alpha_ref * x_hat_ref(ref) + H^T deq(codes_ref)
 * of its neighbour (binary32, in that order: the product, the rotation of the
 * dequantised codes, then their sum), so that decoding loop l reads the codes
 * of every loop between it and the anchor.  Chained policies need every
 * residual loop in one format (same bits, group and rotate; alpha_mode not
 * RQ_ALPHA_ZERO) and num_loops <= 4 (at most RQ_MAX_CHAIN residual loops on a
 * chain); other configurations are RQ_ERR_UNSUPPORTED. */
typedef enum rq_anchor_policy {
  RQ_ANCHOR_LAST = 0,     /* the final loop is every loop's reference (the pages' choice) */
  RQ_ANCHOR_FIRST = 1,    /* loop 0 is every loop's reference */
  RQ_ANCHOR_INTERVAL = 2, /* blocks of anchor_interval loops; each block's last loop
                             (the final loop for a short last block) anchors the block */
  RQ_ANCHOR_PREVIOUS = 3, /* loop l's reference is loop l-1; loop 0 is the anchor */
  RQ_ANCHOR_NEXT = 4      /* loop l's reference is loop l+1; the final loop is the anchor */
} rq_anchor_policy;

/* Longest chain of residual loops a decode call reads (chained policies). */
#define RQ_MAX_CHAIN 3

/* Cache configuration ([RQ] Table 5 caption: loop-wise precision, INT2 with
 * g = 16 or 32, INT4 with g = 32; Figure 1 step 5: mixed precision such as
 * [2,2,2,4]).  Per-loop arrays use entries [0, num_loops).  A zero-filled
 * anchor_policy is the pages' Last-loop reference. */
typedef struct rq_config {
  int32_t num_loops;  /* L in [2, 16] */
  int32_t batch;      /* B >= 1 sequences */
  int32_t kv_heads;   /* Hkv >= 1 */
  int32_t q_heads;    /* Hq = G * Hkv with G in {1, 2, 4, 8} */
  int32_t head_dim;   /* must be RQ_HEAD_DIM */
  int32_t capacity;   /* maximum cached tokens per sequence, >= 1 */
  int32_t bits[RQ_MAX_LOOPS];  /* residual loops: 2 or 4; anchor loops: 16 (bf16) or 4 (INT4) */
  int32_t group[RQ_MAX_LOOPS]; /* residual loops: 16 or 32; anchor loops: 32 (ignored for bf16) */
  int32_t rotate[RQ_MAX_LOOPS];      /* residual loops: 1 = Hadamard-128 rotation, 0 = none; anchors: 0 */
  int32_t alpha_mode[RQ_MAX_LOOPS];  /* residual loops: rq_alpha_mode; anchors: ignored */
  int32_t anchor_policy;    /* rq_anchor_policy */
  int32_t anchor_interval;  /* RQ_ANCHOR_INTERVAL: loops per block, in [2, num_loops] */
} rq_config;

/* Where each plane lives inside the caller's cache buffer.  Every plane is
 * indexed [b][h][t] with t < capacity_padded, one fixed-size record per
 * (b, h, t), and starts on a 1024-byte boundary.  Offsets are bytes from the
 * start of the buffer; -1 marks a plane the configuration does not have.
 * Every loop l has planes codes[l][k|v]; the rest depends on its role:
 *
 *  anchor, bf16:  codes = 128 bf16 per record (256 B); no meta, no alpha
 *  anchor, INT4:  codes = 128 4-bit codes (64 B; element d in bits 4*(d%8) of
 *                 little-endian 32-bit word d/8); meta = 4 groups x (fp16 scale,
 *                 fp16 offset) = 16 B; no alpha
 *  residual:      codes = 128 b-bit codes in the rotated domain (INT2: element d
 *                 in bits 2*(d%16) of word d/16, 32 B; INT4 as above);
 *                 meta = (128/g) x (fp16 scale, fp16 offset);
 *                 alpha = (fp16 alpha_K, fp16 alpha_V) = 4 B
 *  status:        one 32-bit device status word (256 B reserved)
 *  anchor_of[l] is the loop whose anchor planes loop l is decoded against
 *  (anchor_of[l] == l for an anchor loop); ref_of[l] is the loop whose
 *  (reconstructed) values loop l is stored against: anchor_of[l] except under
 *  the chained policies, where it is the neighbouring loop.
 */
typedef struct rq_layout {
  int64_t capacity_padded;
  int64_t total_bytes;
  int64_t status_offset;
  int64_t codes_offset[RQ_MAX_LOOPS][2];
  int64_t meta_offset[RQ_MAX_LOOPS][2];
  int64_t alpha_offset[RQ_MAX_LOOPS];
  int64_t codes_record_bytes[RQ_MAX_LOOPS];
  int64_t meta_record_bytes[RQ_MAX_LOOPS];
  int32_t anchor_of[RQ_MAX_LOOPS];
  int32_t ref_of[RQ_MAX_LOOPS];
} rq_layout;

typedef struct rq_cache rq_cache;

/* Validates cfg and fills *out.  Host only, pure.  RQ_ERR_INVALID_ARG for a
 * null pointer or an out-of-range field; RQ_ERR_UNSUPPORTED for head_dim != 128
 * or a bits/group/G/anchor combination this build does not implement. */
RQ_API rq_status rq_cache_layout(const rq_config* cfg, rq_layout* out);

/* Binds a cache handle to the caller's device buffer (>= layout.total_bytes,
 * 1024-byte aligned) on the current device and zeroes its status word
 * (a synchronous 256-byte cudaMemset).  The buffer stays caller-owned and must
 * outlive the handle.  *out receives a heap-allocated host handle. */
RQ_API rq_status rq_cache_create(const rq_config* cfg, void* device_buffer, int64_t buffer_bytes,
                          rq_cache** out);

/* Frees the host handle only (never the device buffer).  Null is a no-op. */
RQ_API void rq_cache_destroy(rq_cache* cache);

/* Copies the handle's configuration and layout out (either pointer may be null). */
RQ_API rq_status rq_cache_info(const rq_cache* cache, rq_config* cfg_out, rq_layout* layout_out);

/* Encode ([RQ] abstract; Figure 1 steps 2-5): for every loop, sequence b,
 * kv-head h and the n_tokens tokens at positions [pos_b, pos_b + n_tokens):
 * store each anchor loop (bf16 copy or direct INT4 g=32), then for every other
 * loop the fp16 scale alpha against its anchor (LS: <x, ref>/<ref, ref>; norm
 * ratio: ||x||/||ref||; per 128-vector, K and V separately; 0 if ref is 0), the
 * residual x - alpha*ref, its Hadamard-128 rotation and asymmetric min-max group
 * quantisation.  An INT4 anchor's dequantised value is the reference the
 * residuals are taken against.
 *
 *  k, v        device bf16, element [l][b][h][i][d] at
 *              l*strides[0] + b*strides[1] + h*strides[2] + i*strides[3] + d
 *              (strides in elements; d is unit-stride; all strides >= 0)
 *  positions   device int32 [B] start positions, or NULL to use start_pos for
 *              every sequence.  With NULL, start_pos + n_tokens > capacity is
 *              RQ_ERR_CAPACITY; with device positions, tokens past capacity are
 *              skipped and RQ_FLAG_POSITION is set.
 *  n_tokens    >= 0 (0 enqueues nothing).
 * Arithmetic is binary32 with round-to-nearest-even in a fixed order, so codes,
 * scales and offsets are reproducible bit for bit.  Non-finite inputs or
 * |x| > 65504 set RQ_FLAG_BAD_INPUT (their records are then unspecified). */
RQ_API rq_status rq_encode(rq_cache* cache, const void* k, const void* v, const int64_t* strides,
                    int32_t start_pos, const int32_t* positions, int32_t n_tokens,
                    rq_stream_t stream);

/* Decode kernel selection (not a numerical choice: both kernels compute the
 * same attention within the decode tolerance).
 *  RQ_DECODE_KERNEL_SIMT    split kernel on the CUDA cores, 64-token pages
 *                           (128 for the INT4-anchor and anchor-free formats),
 *                           integer dot products for scores and paired fp32
 *                           FMAs for values; every G and every format.
 *  RQ_DECODE_KERNEL_TENSOR  split kernel on the tensor cores (tcgen05), 128-token
 *                           pages: bf16 and int8 MMAs for the scores of all G
 *                           query heads of a kv-head at once and for the
 *                           probability-weighted value sums; G in {1, 2, 4, 8,
 *                           16} (16 rows for some formats: see
 *                           rq_decode_attention_multi); the residual loops of
 *                           chained policies at G in {4, 8} with an INT4
 *                           anchor only.
 *  RQ_DECODE_KERNEL_AUTO    the tensor-core kernel for G >= 4 where it has a
 *                           variant, else the CUDA-core kernel (the default). */
typedef enum {
  RQ_DECODE_KERNEL_AUTO = 0,
  RQ_DECODE_KERNEL_SIMT = 1,
  RQ_DECODE_KERNEL_TENSOR = 2
} rq_decode_kernel;

/* Sets the decode kernel of later rq_decode_attention calls on this handle.
 * RQ_DECODE_KERNEL_TENSOR for a loop format or G it has no variant for makes
 * those calls return RQ_ERR_UNSUPPORTED.  Not thread-safe against concurrent
 * decode calls on the same handle. */
RQ_API rq_status rq_cache_set_decode_kernel(rq_cache* cache, int32_t kernel);

/* Test hook for the failure path (the paper has no counterpart).  With page
 * >= 0, the producer warp of every CTA of later rq_decode_attention calls on
 * this handle waits, before issuing its page-th page, on a barrier that nothing
 * arrives at.  That wait, like every wait in the decode kernels, gives up after
 * its limit (about 2 s); the call then completes with RQ_FLAG_PIPE_TIMEOUT set
 * in the status word (its output is unspecified) and the context stays usable.
 * -1 (the default) turns the hook off; other values are RQ_ERR_INVALID_ARG. */
RQ_API rq_status rq_cache_set_debug_stall(rq_cache* cache, int32_t page);

/* Bytes of workspace rq_decode_attention needs for this cache on the current
 * device (split-K partials; independent of context length). */
RQ_API rq_status rq_decode_workspace_size(const rq_cache* cache, int64_t* bytes_out);

/* Fused decode attention of one loop over the compact cache
 * ([RQ] abstract: "reduced KV memory traffic"; Figure 1).  For a residual loop
 * each cached token t < ctx_len[b] scores
 *     s_t = softmax_scale * ( alpha_K,t (q . ref_k,t) + (H q) . deq(codes_K,t) )
 * and the output is
 *     ( sum_t p_t alpha_V,t ref_v,t  +  H^T sum_t p_t deq(codes_V,t)
 *       + sum_tail p_j v_tail,j ) / sum p
 * with one inverse rotation per (b, q-head), ref being the loop's anchor.  Under
 * a chained policy the loop's chain l = c_0 -> c_1 -> ... -> anchor unrolls to
 *     s_t = softmax_scale * ( beta_n (q . ref_k) + sum_i beta_i (H q) . deq(codes_K of c_i) )
 * with beta_0 = 1 and beta_(i+1) = beta_i * alpha_K of c_i per token (alpha_V
 * likewise for the value sums); it runs on the CUDA-core kernel only.  An
 * anchor loop is plain attention over its bf16 or INT4 planes.  n_tail current tokens (bf16,
 * not yet encoded) join the softmax.  Split-K over pages (64 or 128 tokens on
 * the CUDA-core kernel, 128 on the tensor-core kernel) with an online softmax,
 * merged by a second kernel.
 *
 *  q          device bf16 [B][Hq][128]
 *  ctx_len    device int32 [B], each in [0, capacity] (clamped, RQ_FLAG_CTX_LEN)
 *  k_tail/v_tail  device bf16 [B][Hkv][n_tail][128] (NULL allowed when n_tail == 0)
 *  softmax_scale  e.g. 1/sqrt(128)
 *  out        device fp32 [B][Hq][128]; kv-head of q-head j is j / G
 *  workspace  device, >= rq_decode_workspace_size bytes, 256-byte aligned */
RQ_API rq_status rq_decode_attention(const rq_cache* cache, int32_t loop, const void* q,
                              const int32_t* ctx_len, const void* k_tail, const void* v_tail,
                              int32_t n_tail, float softmax_scale, float* out, void* workspace,
                              int64_t workspace_bytes, rq_stream_t stream);

/* Largest number of draft tokens of one rq_decode_attention_multi call. */
#define RQ_MAX_DRAFT 16

/* Bytes of workspace rq_decode_attention_multi needs for n_q draft tokens
 * (n_q in [1, RQ_MAX_DRAFT]). */
RQ_API rq_status rq_decode_multi_workspace_size(const rq_cache* cache, int32_t n_q, int64_t* bytes_out);

/* Multi-query decode: rq_decode_attention for n_q query tokens per sequence at
 * once, as when a decoding model verifies n_q draft tokens (speculative
 * decoding) or decodes several positions in one step.  The paper has no
 * counterpart; it widens the same computation.  Draft token i (0-based) of
 * sequence b attends to the ctx_len[b] cached tokens and to tail tokens
 * 0 .. n_tail - n_q + i: the last n_q tail tokens are the draft tokens' own
 * keys and values (bf16, not yet encoded), each visible to itself and to the
 * later ones, and any earlier tail tokens to all.  Up to 8 query rows per
 * kv-head (n_q * G) share every read of its cached pages, and 16 rows do where
 * the tensor-core kernel has a 16-row variant for the loop's format (residuals
 * in 32-dim groups with an INT4 anchor or none, INT2 g=32 residuals with a bf16
 * anchor, and both anchor loops) and the call takes that kernel; other rows run
 * in blocks of 16 or 8, one pass over the cache each.  With 4 or more rows in a
 * block the automatic kernel choice is the tensor-core kernel.
 *  q        device bf16 [B][n_q][Hq][128]
 *  out      device fp32 [B][n_q][Hq][128]
 *  n_q      in [1, RQ_MAX_DRAFT] (else RQ_ERR_INVALID_ARG) with n_q * (Hq / Hkv)
 *           in {1, 2, 4} or a multiple of 8 (else RQ_ERR_UNSUPPORTED)
 *  n_tail   >= n_q when n_q > 1 (RQ_ERR_INVALID_ARG otherwise)
 *  workspace  >= rq_decode_multi_workspace_size(cache, n_q) bytes
 * Other arguments, layouts and errors as rq_decode_attention (which is n_q = 1). */
RQ_API rq_status rq_decode_attention_multi(const rq_cache* cache, int32_t loop, const void* q, int32_t n_q,
                                           const int32_t* ctx_len, const void* k_tail, const void* v_tail,
                                           int32_t n_tail, float softmax_scale, float* out, void* workspace,
                                           int64_t workspace_bytes, rq_stream_t stream);

/* How rq_decode_attention_multi (n_q draft tokens; rq_decode_attention is
 * n_q = 1) would run `loop` on this handle, without running it: the kernel it
 * takes (RQ_DECODE_KERNEL_SIMT or RQ_DECODE_KERNEL_TENSOR) and the query rows
 * per kv-head of one pass over the cache; n_q * G / rows_per_pass passes read
 * the loop's pages.  Returns what that call would return for an unsupported
 * loop, n_q or kernel (RQ_ERR_INVALID_ARG, RQ_ERR_UNSUPPORTED).  Host only. */
RQ_API rq_status rq_decode_plan(const rq_cache* cache, int32_t loop, int32_t n_q, int32_t* kernel_out,
                                int32_t* rows_per_pass_out);

/* rq_decode_attention of `loop`, plus the encode of n_new new tokens of every
 * loop into the cache in the same call: the per-step append of a decoding
 * model ([RQ] abstract; Figure 1 steps 2-5), which can run once the final
 * loop has produced its keys and values, so it is typically fused into the
 * final loop's decode.  The encode runs in the launch of the combine kernel,
 * by extra warps, saving one launch per layer and step.
 *  k_new/v_new, strides   as rq_encode (all loops; n_new tokens)
 *  positions              device int32 [B], required: sequence b's new tokens go
 *                         to positions[b] .. positions[b] + n_new - 1; positions
 *                         past capacity are skipped with RQ_FLAG_POSITION
 * The decode reads positions < ctx_len[b] only: to append the current token,
 * pass positions = ctx_len (its values join this decode through the tail).
 * Arithmetic and results are those of rq_decode_attention followed by
 * rq_encode with device positions. */
RQ_API rq_status rq_decode_attention_append(rq_cache* cache, int32_t loop, const void* q,
                                            const int32_t* ctx_len, const void* k_tail, const void* v_tail,
                                            int32_t n_tail, float softmax_scale, float* out, void* workspace,
                                            int64_t workspace_bytes, const void* k_new, const void* v_new,
                                            const int64_t* strides, const int32_t* positions, int32_t n_new,
                                            rq_stream_t stream);

/* Size of the library's static split-K scratch used by
 * rq_decode_attention_static_scratch (4 MiB). */
#define RQ_STATIC_SCRATCH_BYTES (4u * 1024u * 1024u)

/* rq_decode_attention for callers that cannot allocate device memory.  The
 * paper has no counterpart of this entry point: it exists for callers that have
 * no way to provide the decode workspace, such as code hosted in a framework
 * that owns every device allocation and forbids raw cudaMalloc, or serving
 * loops that must not allocate while running (cudaMalloc and cudaFree can
 * synchronise the device).  It computes exactly what rq_decode_attention
 * computes, with the split-K partials kept in a fixed RQ_STATIC_SCRATCH_BYTES
 * array in the library's own device memory instead of a caller workspace.
 *  - It allocates nothing and calls no allocating routine.
 *  - Limit: the split-K partials of this decode must fit in
 *    RQ_STATIC_SCRATCH_BYTES: (batch*kv_heads + SMs) * G * 1040 bytes, with G
 *    the query rows of one pass over the cache (q_heads / kv_heads up to 8; 16
 *    where a 16-row tensor-core pass takes them, else 8; 4 where the default
 *    decode runs 8 rows as two passes of 4); otherwise it returns
 *    RQ_ERR_WORKSPACE before enqueuing anything.
 *  - Device: the device current at the call must be the one the cache was
 *    created on (RQ_ERR_INVALID_ARG otherwise).
 *  - Set-up: the first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  Every GPU that loads the library keeps the
 *    array until the process exits.
 *  - Sharing: all calls on a device use the same array, which keeps the last
 *    call's contents (nothing in it needs to start at zero).  Calls whose
 *    kernels overlap on the GPU -- on different streams, or from different
 *    host threads -- race on it; serialise them on one stream.
 * Arguments and errors are those of rq_decode_attention, minus the workspace. */
RQ_API rq_status rq_decode_attention_static_scratch(const rq_cache* cache, int32_t loop, const void* q,
                                                    const int32_t* ctx_len, const void* k_tail,
                                                    const void* v_tail, int32_t n_tail, float softmax_scale,
                                                    float* out, rq_stream_t stream);

/* Workspace bytes for rq_bf16_decode_attention with these sizes. */
RQ_API rq_status rq_bf16_decode_workspace_size(int32_t batch, int32_t kv_heads, int32_t q_heads,
                                        int64_t* bytes_out);

/* Decode attention over a plain bf16 KV cache (the BF16-cache baseline the
 * [RQ] abstract compares against; same kernels with no residual):
 *  k_cache/v_cache  device bf16, element [b][h][t][d] at b*strides[0] +
 *                   h*strides[1] + t*strides[2] + d (strides in elements,
 *                   multiples of 8, base 16-byte aligned), t < capacity
 *  other arguments as rq_decode_attention; status flags go to *status_word if
 *  it is non-null (device int32), else are dropped. */
RQ_API rq_status rq_bf16_decode_attention(int32_t batch, int32_t kv_heads, int32_t q_heads,
                                   const void* k_cache, const void* v_cache,
                                   const int64_t* strides, int32_t capacity, const void* q,
                                   const int32_t* ctx_len, const void* k_tail, const void* v_tail,
                                   int32_t n_tail, float softmax_scale, float* out,
                                   void* workspace, int64_t workspace_bytes, int32_t* status_word,
                                   rq_stream_t stream);

/* Reconstruction (test support): fp32 K_hat, V_hat of loop `loop` for tokens
 * [t0, t0 + n) of every (b, h), written to k_out/v_out [B][Hkv][n][128]:
 * alpha * ref + H^T deq(codes) for a residual loop, the (dequantised)
 * anchor for an anchor loop.  Under a chained policy ref is the reconstruction
 * of the loop's reference, computed in the same buffers from the anchor
 * outward (one launch per loop of the chain). */
RQ_API rq_status rq_reconstruct(const rq_cache* cache, int32_t loop, int32_t t0, int32_t n, float* k_out,
                         float* v_out, rq_stream_t stream);

/* Synchronises `stream`, reads and clears the device status word.  Returns
 * RQ_OK if it was zero, else RQ_ERR_DEVICE_FLAG with the bits in *flags_out
 * (may be null). */
RQ_API rq_status rq_get_error(const rq_cache* cache, rq_stream_t stream, uint32_t* flags_out);

/* Static string naming a status code. */
RQ_API const char* rq_status_string(rq_status status);

/* Detail of the calling thread's most recent non-OK status ("" if none). */
RQ_API const char* rq_last_error_message(void);

#ifdef __cplusplus
}
#endif
#endif /* RQ_API_H */
