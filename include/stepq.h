/*
 * stepq.h -- C ABI of libstepq: the decode step of a gated Delta-rule layer whose
 * per-request d_k x d_v state is stored quantized (STEPQuant), for NVIDIA B200 (sm_100a).
 *
 * Sources, by page title and section (web pages on STEPQuant, arXiv 2609.38169):
 *   [SUM]  hyper.ai paper summary, "Method" (symmetric uniform state quantization applied
 *          after the update and the readout; lifetime-aware bit allocation; key-row-aware
 *          dual-axis fitting; packed-state kernels on a recurrent-state pool)
 *   [EXP]  "Paper Explained: STEPQuant -- When and Where Quantization Errors Matter in
 *          Delta-Rule Recurrent States", "The mechanism: rewriting state with the delta rule"
 *   [BLOG] ONTLE blog post on STEPQuant: per-request state pool with pre-allocated spare
 *          slots; bit allocation, pivots and impact scores fixed offline, dual-axis scales
 *          refit at every decoding step; the fused decode kernel
 *
 * Conventions
 *   - Every function returns a status (stepq_status); 0 is success.
 *   - A pool owns its device memory.  The caller owns every other buffer.  Unless stated
 *     otherwise, tensor arguments are DEVICE pointers to contiguous row-major arrays, and
 *     must be 16-byte aligned.
 *   - Calls that take a stream enqueue work on it and return without synchronizing; an
 *     asynchronous CUDA fault surfaces as STEPQ_CUDA_ERROR on a later call.  A pool must
 *     not be used on two streams at once without synchronization by the caller.
 *   - slot_ids within one call must be distinct; duplicates give undefined results (the
 *     debug mode of stepq_pool_set_debug rejects them).  An out-of-range slot id is skipped by
 *     the kernels and raises the pool's sticky device flag (read with stepq_pool_get_error);
 *     kernels never trap.
 *   - Each data-path call (load, dump, decode) opens an NVTX range named after itself over its
 *     argument checks and enqueue, so a profiler that records NVTX can attribute the call's
 *     kernels to it; with no tool attached this costs a few nanoseconds.
 *
 * State and layout (shared by every call; the pages leave the format open)
 *   - value head h of request b lives in slot s = slot_ids[b]; key head g(h) = h / (H / H_k)
 *   - the pool is slot-major; inside a slot the value heads follow in order; a head block is
 *       codes | r[d_k] float32 | c[d_v] float32
 *     with the head's bit width b in {4, 6, 8}; block sizes 9216, 13312, 17408 bytes for
 *     d_k = d_v = 128 (all multiples of 128 bytes)
 *   - a state is S_ij ~= Q_ij * r_i * c_j with integer codes |Q_ij| <= qmax = 2^(b-1) - 1
 *   - codes are stored as offset binary u = Q + 2^(b-1) in a little-endian bit stream of
 *     b-bit fields (4-bit: two per byte, low nibble first; 6-bit: four per three bytes;
 *     8-bit: one per byte); the element order in the stream is panel-major: 16-column
 *     panels, each panel row-major, i.e. stream index = (j / 16) * d_k * 16 + i * 16 + j % 16
 *   - a zero-filled block (r = c = 0) is the zero state
 *   - FP16 pivot heads (width 16; STEPQuant summary, "Method" para 2: the highest-risk
 *     units are kept in FP16 as sparse pivots): the block is the state itself, d_k x d_v
 *     IEEE binary16 values, row-major, little-endian (32768 bytes), no scales; each step
 *     stores the updated state rounded to binary16 (nearest, ties to even)
 */
#ifndef STEPQ_H
#define STEPQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STEPQ_API __attribute__((visibility("default")))
#else
#define STEPQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* same type as cudaStream_t; NULL = legacy stream */
typedef struct CUstream_st *stepq_stream;

typedef enum {
    STEPQ_OK = 0,
    STEPQ_INVALID_ARG = -1,              /* null pointer, bad size or alignment, bad count   */
    STEPQ_OUT_OF_MEMORY = -2,            /* device or host allocation failed                 */
    STEPQ_CUDA_ERROR = -3,               /* a CUDA runtime call or kernel launch failed      */
    STEPQ_UNSUPPORTED = -4,              /* d_k or d_v != 128, or a width not in {4,6,8,16}  */
    STEPQ_DEVICE_FLAG = -5               /* the pool's sticky device flag was set            */
} stepq_status;

enum { STEPQ_GATE_GDN = 0, STEPQ_GATE_KDA = 1 };
enum { STEPQ_DTYPE_F32 = 0, STEPQ_DTYPE_BF16 = 1 };

/* Bits of the sticky device flag. */
enum {
    STEPQ_FLAG_BAD_SLOT = 1,             /* a slot id outside [0, num_slots) was skipped     */
    STEPQ_FLAG_TIMEOUT = 2               /* a bounded wait inside a kernel gave up           */
};

typedef struct stepq_pool stepq_pool;

typedef struct {
    int32_t num_slots;                   /* pool slots (requests resident at once + spares)  */
    int32_t num_heads;                   /* value heads H                                    */
    int32_t num_key_heads;               /* key heads H_k, divides H                         */
    int32_t d_k, d_v;                    /* state shape; 128 x 128 is supported              */
    int32_t gate_mode;                   /* STEPQ_GATE_GDN: alpha [n, H];
                                            STEPQ_GATE_KDA: alpha [n, H, d_k]                 */
    int32_t in_dtype;                    /* STEPQ_DTYPE_F32 or _BF16: dtype of q, k, v,
                                            alpha and beta (y is always float32)             */
    const uint8_t *head_bits;            /* HOST array [H], each 4, 6, 8 or 16 (16: an FP16
                                            pivot head; from an offline allocation, e.g.
                                            stepq_allocate_bits_pivots)                      */
} stepq_pool_desc;

/* Create a pool and zero it (every slot holds the zero state).  The descriptor and
 * head_bits are copied.  Synchronizes the device.  [BLOG: pool with spare slots] */
STEPQ_API int stepq_pool_create(const stepq_pool_desc *desc, stepq_pool **out);

/* Pool whose heads of width 0 carry per-key-row widths.      [BLOG: the allocation unit of
 * Kimi's KDA is a single key row]  desc as for stepq_pool_create, except that head_bits[h]
 * may be 0; row_bits (HOST [H, d_k], entries in {4, 6, 8}) then gives the width of each key
 * row of head h (entries of other heads are ignored).  Such a head stores its rows grouped
 * by width -- 8-bit rows, then 4-bit, then 6-bit, each group in ascending key-row order --
 * with each 16-column panel holding one segment of 16 codes per stored row at the row's
 * width, padded to a multiple of 16 bytes; then r[d_k] in stored-row order, then c[d_v].
 * Block bytes = 8 * roundup16(16 n8 + 8 n4 + 12 n6) + 4 d_k + 4 d_v.  The fit is the clip-free
 * fit at each row's own levels (qmax = 2^(b_i - 1) - 1); the impact-weighted fit
 * (stepq_pool_set_impact) applies to the heads of uniform width only.  The allocation-free
 * entry point does not take such pools. */
STEPQ_API int stepq_pool_create_rows(const stepq_pool_desc *desc, const uint8_t *row_bits, stepq_pool **out);

/* Free the pool and its device memory.  Synchronizes the device.  NULL is a no-op. */
STEPQ_API int stepq_pool_destroy(stepq_pool *pool);

/* Bytes of one slot and of the whole pool (host outputs; either may be NULL). */
STEPQ_API int stepq_pool_bytes(const stepq_pool *pool, size_t *slot_stride, size_t *total);

/* Byte offset of value head h's block inside a slot (host output). */
STEPQ_API int stepq_pool_head_offset(const stepq_pool *pool, int32_t h, size_t *offset);

/* Quantize fp32 states into slots: S [n, H, d_k, d_v] float32 (device).  Per state:
 * clip-free dual-axis fit c_j = sqrt(max_i |S_ij|), r_i = max_j (|S_ij| / c_j) / qmax,
 * then Q_ij = nearest level of S_ij / (r_i c_j), ties to even.  [SUM Method: fitting] */
STEPQ_API int stepq_pool_load_fp32(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const float *S,
                         stepq_stream stream);

/* Copy packed slot images into slots: bytes [n, slot_stride] (device), e.g. from
 * stepq_pool_dump_packed or a checkpoint.  Restores states bit for bit. */
STEPQ_API int stepq_pool_load_packed(stepq_pool *pool, const int32_t *slot_ids, int32_t n,
                           const uint8_t *bytes, stepq_stream stream);

/* Dequantize slots: S_out [n, H, d_k, d_v] float32 (device), S_ij = Q_ij * r_i * c_j. */
STEPQ_API int stepq_pool_dump_fp32(const stepq_pool *pool, const int32_t *slot_ids, int32_t n, float *S_out,
                         stepq_stream stream);

/* Copy slot images out: bytes_out [n, slot_stride] (device). */
STEPQ_API int stepq_pool_dump_packed(const stepq_pool *pool, const int32_t *slot_ids, int32_t n,
                           uint8_t *bytes_out, stepq_stream stream);

/* One decode step for n requests, every value head, in one fused kernel.
 * Per (request b, value head h), with S the state in slot slot_ids[b]:
 *   dequantize S_ij = Q_ij r_i c_j;  fade S'_ij = alpha_i S_ij (GDN: one alpha per head;
 *   KDA: one per key channel);  predict u = S'^T k;  write S = S' + k (beta (v - u))^T;
 *   read y = S^T q from the updated, unquantized state;  refit r, c;  requantize to the
 *   head's width with round-half-even;  repack in place.       [EXP mechanism; SUM Method]
 * Arguments (device, in_dtype unless noted):
 *   q, k   [n, H_k, d_k]     query and key (used as given: no normalization or scaling)
 *   v      [n, H, d_v]
 *   alpha  [n, H] (GDN) or [n, H, d_k] (KDA): retention in (0, 1], not its logarithm
 *   beta   [n, H]
 *   y      [n, H, d_v] float32 output; rows of skipped (bad-slot) requests are not written
 * n = 0 is a valid no-op.  In a pool with FP16 pivot heads their kernel runs on a stream of
 * the pool, forked from `stream` at the call and joined back to it: work enqueued on `stream`
 * after the call sees every head updated.  The call may be captured in a CUDA graph. */
STEPQ_API int stepq_decode_step(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const void *q,
                      const void *k, const void *v, const void *alpha, const void *beta, float *y,
                      stepq_stream stream);

/* The decode step of stepq_decode_step with every per-step buffer in HOST memory: the call
 * copies slot_ids and the inputs into a device staging buffer owned by the pool, runs the
 * step, and copies y back.  The paper has no counterpart to this entry point; it is the
 * path of a caller whose tokens arrive in host memory.  All of it is asynchronous:
 *   slot_ids [n] int32, q, k, v, alpha, beta   HOST, layouts and dtypes as for stepq_decode_step
 *   y        HOST [n, H, d_v] float32, written when the call's copy-out runs
 * The pool keeps two staging buffers and uses them in turn; the inputs are copied on a
 * copy-in stream of the pool, the step runs on `stream`, and y is copied on a copy-out stream
 * of the pool, chained by events, so the copies of consecutive calls overlap the steps of
 * their neighbours.  Host buffers must stay valid and unchanged (inputs), or unread (y),
 * until the call's copies are done: after stepq_pool_host_wait(pool, s) and a
 * synchronization of s.  Page-locked host memory lets the copies run asynchronously;
 * pageable memory works, with copies that hold up the calling thread.  The first call, and a
 * call with more requests than any before it, allocates the staging buffers (a regrowth first
 * waits for the copies of the earlier calls).  A pool must not be used from several host
 * threads at once.  Errors: as for stepq_decode_step; argument checks come before any copy. */
STEPQ_API int stepq_decode_step_host(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const void *q,
                                     const void *k, const void *v, const void *alpha, const void *beta, float *y,
                                     stepq_stream stream);

/* Layout of a contiguous host input image for stepq_decode_step_host: for n requests of this
 * pool, offsets_out[0..5] (HOST, 6 entries) receive the byte offsets of slot_ids, q, k, v,
 * alpha and beta from the start of the image (slot_ids at 0, each a multiple of 256 bytes,
 * each array as laid out for stepq_decode_step), and total_out (may be NULL) the image's
 * size.  When a call's six host inputs sit at exactly these offsets of one buffer (slot_ids
 * at its start), the call copies them to the device as one transfer instead of six; any
 * other placement works as before.  The paper has no counterpart. */
STEPQ_API int stepq_host_image_layout(const stepq_pool *pool, int32_t n, size_t *offsets_out, size_t *total_out);

/* Makes `stream` wait for every copy that stepq_decode_step_host calls on this pool have
 * enqueued, y included.  Enqueues only; synchronize `stream` to wait on the host. */
STEPQ_API int stepq_pool_host_wait(stepq_pool *pool, stepq_stream stream);

/* The decode step of stepq_decode_step for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point.  Some callers may not call cudaMalloc:
 * code running inside a serving engine or framework that owns all device memory through
 * its own arena or caching allocator (and accounts for every byte), or code embedded where
 * new allocations are forbidden.  They keep the packed state themselves and pass it here;
 * no pool object exists.
 *   desc      as for stepq_pool_create (HOST, read during the call), with two limits that
 *             give STEPQ_UNSUPPORTED: num_heads <= 256 (the scratch holds the tables of at
 *             most 256 heads), and every head_bits[h] in {4, 6, 8} (FP16 pivot heads, width
 *             16, are not taken: their kernel runs on a second stream of a pool)
 *   state     DEVICE, caller-owned, 128-byte aligned: num_slots slots in the pool layout
 *             (slot_stride = sum of the head block sizes), updated in place
 *   slot_ids, q, k, v, alpha, beta, y   as for stepq_decode_step
 *   flag_out  DEVICE, optional (may be NULL): receives this call's STEPQ_FLAG_* bits
 * The kernel's scratch (the flag word and the per-head tables, 3584 bytes) is a fixed device
 * array inside the library, held by every GPU that loads it until the process exits.  Every
 * call rewrites it (flag cleared, tables refreshed) on `stream`, with a one-CTA kernel that
 * receives the new contents as its launch argument, so the call reads no host memory
 * asynchronously and does not wait on the host for earlier work of `stream`.  Calls that
 * overlap on the GPU (other streams, other threads) share the array and race.  The first call
 * on each device resolves the array's address and configures the kernels on that device,
 * so it should come before any stream capture.  The call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine). */
STEPQ_API int stepq_decode_step_noalloc(const stepq_pool_desc *desc, uint8_t *state, const int32_t *slot_ids,
                                        int32_t n, const void *q, const void *k, const void *v,
                                        const void *alpha, const void *beta, float *y, int32_t *flag_out,
                                        stepq_stream stream);

/* Key-row-aware dual-axis fitting with row-impact scores.          [SUM Method, paras 3-4; BLOG]
 * impact: HOST [H, d_k] float32 row-impact scores (positive, finite; fixed offline, e.g. the
 * expected squared readout weight of each key row over calibration tokens), or NULL to
 * return to the clip-free fit.  Each head's scores are normalized to mean 1
 * (w_i = float(omega_i / mean(omega)), in double).  While set, stepq_pool_load_fp32 and
 * stepq_decode_step fit every quantized head of the pool as (S: the updated state in fp32):
 *   r_i  = sqrt(max_j |S_ij| / w_i)                      row: magnitude against impact
 *   c0_j = max_i (|S_ij| / r_i) / qmax,  Q0 = nearest levels of S / (r c0)
 *   c_j  = sum_i w_i r_i Q0_ij S_ij / sum_i w_i r_i^2 Q0_ij^2   (c0_j if a sum is <= 0)
 *   Q    = nearest levels of S / (r c), clipped to [-qmax, qmax]
 * FP16 pivot heads are unaffected.  Synchronizes the device; STEPQ_INVALID_ARG for a
 * non-positive or non-finite score. */
STEPQ_API int stepq_pool_set_impact(stepq_pool *pool, const float *impact);

/* Health check of the kernels' failure path: a one-warp kernel waits on a shared-memory
 * barrier that nothing completes (no copy in flight), with the same bounded wait as the
 * decode kernel but a short poll limit, then raises STEPQ_FLAG_TIMEOUT and exits.  flag_out
 * (HOST) receives the flag bits: STEPQ_FLAG_TIMEOUT when the path works.  The context stays
 * usable.  Synchronizes `stream`. */
STEPQ_API int stepq_check_wait_timeout(int32_t *flag_out, stepq_stream stream);

/* Debug checks of a pool, off by default.  With STEPQ_DEBUG_SLOTS, every call of the pool that
 * takes slot_ids rejects duplicate or out-of-range ids with STEPQ_INVALID_ARG before any
 * device work (without it, duplicates give undefined results and an out-of-range id is
 * skipped by the kernels and flagged).  For device slot_ids the check copies them to the host
 * and synchronizes the call's stream, so a pool in this mode is for development runs, not for
 * stream capture; stepq_decode_step_host checks its host ids directly.  flags = 0 turns the
 * checks off; unknown flag bits give STEPQ_INVALID_ARG.  The paper has no counterpart. */
enum { STEPQ_DEBUG_SLOTS = 1 };
STEPQ_API int stepq_pool_set_debug(stepq_pool *pool, int32_t flags);

/* The same check on a HOST array: STEPQ_OK when slot_ids[0 .. n) are distinct and each lies in
 * [0, num_slots), else STEPQ_INVALID_ARG (also for n < 0, num_slots <= 0, or a null array
 * with n > 0).  Reads the array only; no device work.  The paper has no counterpart. */
STEPQ_API int stepq_check_slot_ids(const int32_t *slot_ids, int32_t n, int32_t num_slots);

/* Read and clear the pool's sticky device flag (host output, STEPQ_FLAG_* bits).
 * Synchronizes the device. */
STEPQ_API int stepq_pool_get_error(stepq_pool *pool, int32_t *flag_out);

/* Lifetime-aware bit allocation (host, offline).             [SUM Method, para 2; BLOG]
 * For each unit u (a head): retention rho_u = 2^(-1 / half_life[u]) (the mean log
 * retention of the unit), lifetime weight w_u = 1 / (1 - rho_u) (error retention after j
 * updates ~ rho^j, summed); distortion D_u(b) = distortion[u * C + c] for candidate
 * cand[c], or, when distortion is NULL, 2^(-2 b) (a uniform quantizer's error power).
 * Chooses bits_out[u] in cand minimising sum_u w_u D_u(bits_out[u]) subject to
 * sum_u bits_out[u] <= floor(N * avg_bits), by exact dynamic programming.
 * All pointers are HOST pointers.  half_life must be finite and > 0; cand must be
 * distinct widths in {4, 6, 8}.  Returns STEPQ_INVALID_ARG when no assignment fits. */
STEPQ_API int stepq_allocate_bits(const double *half_life, const double *distortion, int32_t N,
                        const uint8_t *cand, int32_t C, double avg_bits, uint8_t *bits_out);

/* Lifetime-aware allocation with FP16 pivots (host, offline).  [SUM Method, para 2]
 * The n_pivots units of highest risk w_u * D_u(b_max) (b_max the widest candidate; ties go
 * to the lower index) get width 16 and sit outside the budget; the other N - n_pivots units
 * are allocated as by stepq_allocate_bits with the budget floor((N - n_pivots) * avg_bits).
 * Returns STEPQ_INVALID_ARG also for n_pivots outside [0, N]. */
STEPQ_API int stepq_allocate_bits_pivots(const double *half_life, const double *distortion, int32_t N,
                                         const uint8_t *cand, int32_t C, double avg_bits, int32_t n_pivots,
                                         uint8_t *bits_out);

/* Static description of a status code. */
STEPQ_API const char *stepq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* STEPQ_H */
