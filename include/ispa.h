/*
 * ispa.h -- C ABI of libispa, the B200 (sm_100a) implementation of the warmup-phase hot
 * path of Instance-Specific Parametric Absorption (ISPA).
 *
 * Source of the method: "Towards Memory-Efficient Autoregressive Video Generation via
 * Instance-Specific Parametric Absorption", paper text (paperpeel.com/paper/2607.00712),
 * cited as [ISPA §x]; the reading notes at paper.gecl.asia, section "Method", cited as
 * [notes: Method]. The paper publishes no API; these calls follow its problem statement.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Memory: the caller owns every buffer. Pointers named "device" must be device memory
 *    of the current CUDA device; "host" pointers are host memory. The library allocates
 *    nothing; calls that need scratch space take a caller-provided workspace `ws` of at
 *    least ispa_workspace_bytes(...) bytes (256-byte aligned).
 *  - Layouts (row-major): Q, K, V, O are [rows, heads, head_dim]; KV rows are in time
 *    order. An attention output seen as a matrix A is [n_q, D] with D = heads*head_dim and
 *    column h*head_dim + j. W (the attention output projection) is stored [D_in, D_out]
 *    so that y = A W; a torch nn.Linear weight is its transpose. The bias of the
 *    projection cancels out of the residual and is not used.
 *  - lse arrays are [heads, n_q] float32, natural logarithm of the softmax denominator of
 *    scale * q.k over the partition; an empty partition has lse = -inf and output 0.
 *  - dtype ISPA_BF16: Q/K/V/O/W in bf16, softmax and accumulation in float32, the
 *    statistics operands A_loc and R rounded to bf16, statistics in float32.
 *    dtype ISPA_FP32: everything in float32.
 *  - Asynchrony: every device call is enqueued on `stream` (NULL = legacy default
 *    stream) and returns before the GPU finishes. Argument errors are reported before
 *    anything is enqueued; a launch failure returns ISPA_ERR_CUDA. Errors found on the
 *    device (a bounded wait that ran out) are latched in a per-device flag that
 *    ispa_device_status() reads and clears.
 *  - Threading: calls may come from several host threads; ispa_last_error() is
 *    per-thread.
 *  - Device reset: the library looks up the device address of each of its own device
 *    variables (the error flag; the static scratch of ispa_attn_split_noalloc) once per device
 *    and keeps it for the life of the process. cudaDeviceReset frees them: after resetting a
 *    device, make no further library call on that device in the same process.
 */
#ifndef ISPA_H
#define ISPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ispa_stream_t; /* a cudaStream_t */

typedef enum {
    ISPA_OK = 0,
    ISPA_ERR_INVALID_ARG = -1,  /* bad pointer, size, range or dtype; nothing enqueued  */
    ISPA_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. head_dim not 64/128) */
    ISPA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed                     */
    ISPA_ERR_NOT_SPD = -4,      /* G + lambda*I was not positive definite for a layer    */
    ISPA_ERR_TIMEOUT = -5,      /* a bounded device-side wait ran out (device flag)      */
    ISPA_ERR_WORKSPACE = -6     /* ws is NULL, misaligned or smaller than required       */
} ispa_status;

typedef enum { ISPA_BF16 = 0, ISPA_FP32 = 1 } ispa_dtype;

/* One layer's attention call. The KV rows [0, n_kv) split into two partitions
 * [ISPA §3.1 step 1]: the local partition = [sink_begin, sink_end) U [chunk_begin,
 * chunk_end) (sink frame + current chunk), and the history partition = every other row.
 * Ranges may be empty; they must lie inside [0, n_kv) and must not overlap. */
typedef struct {
    int n_q;          /* query rows (tokens of the chunk)                  */
    int n_kv;         /* cached KV rows, sink and chunk included           */
    int heads;        /* attention heads                                   */
    int head_dim;     /* 64 or 128                                         */
    int sink_begin, sink_end;
    int chunk_begin, chunk_end;
    float scale;      /* softmax scale, normally 1/sqrt(head_dim)          */
    ispa_dtype dtype;
} ispa_attn_desc;

/* Ridge statistics of one layer [ISPA §3.2; notes: Method], all device memory:
 * G = sum A_loc^T A_loc, C = sum A_loc^T R, H = sum R^T R (R = A_full - A_loc), each
 * [D, D] float32 row-major, and rows = number of token rows accumulated. */
typedef struct {
    int D;
    float *G;
    float *C;
    float *H;
    long long *rows;
} ispa_stats;

/* ispa_attn_split -- decomposable attention [ISPA §3.1 step 1 "Dual-Stream Warmup",
 * §3.4 "Decomposable Attention"]: one pass over the KV rows gives the local output
 * (O_loc, lse_loc) and the history output (O_hist, lse_hist), merged by their
 * log-sum-exps into the full output: lse_full = logaddexp(lse_loc, lse_hist),
 * O_full = e^(lse_loc-lse_full) O_loc + e^(lse_hist-lse_full) O_hist.
 *   q [n_q, heads, head_dim], k/v [n_kv, heads, head_dim]     (device, dtype)
 *   o_full [n_q, heads, head_dim] (device, dtype), lse_full [heads, n_q] (device)
 *   o_loc/lse_loc/o_hist/lse_hist: optional outputs (NULL to skip)
 *   stats: optional; when given, R = O_full - O_loc is formed on chip and
 *     G += A_loc^T A_loc, C += A_loc^T R, H += R^T R, rows += n_q (fused accumulation,
 *     [ISPA §3.2]); stats->D must equal heads*head_dim. With stats == NULL the call is
 *     plain full attention (an F-layer after the switch [ISPA §3.1 step 3]).
 *   ws: workspace of ispa_workspace_bytes(desc, 1, D) bytes when stats != NULL
 *     (may be NULL otherwise). */
int ispa_attn_split(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                    void *o_full, float *lse_full, void *o_loc, float *lse_loc, void *o_hist,
                    float *lse_hist, const ispa_stats *stats, void *ws, size_t ws_bytes,
                    ispa_stream_t stream);

/* ispa_attn_split_ops -- ispa_attn_split without the accumulation: the call's statistics
 * operands A_loc and R = A_full - A_loc (computed on chip from the partition outputs, then
 * rounded to desc->dtype) are written to a_ops and r_ops, each [n_q, heads*head_dim] device
 * memory of desc->dtype, 16-byte aligned. With ispa_accum_ops this splits a warmup chunk into
 * the attention of every layer followed by one statistics launch for all of them. */
int ispa_attn_split_ops(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                        void *o_full, float *lse_full, void *o_loc, float *lse_loc, void *o_hist,
                        float *lse_hist, void *a_ops, void *r_ops, ispa_stream_t stream);

/* ispa_accum_ops -- G += A^T A, C += A^T R, H += R^T R and rows += n_rows for n_layers layers
 * [ISPA §3.2]: a_ops and r_ops hold the layers' operands one after the other
 * ([n_layers][n_rows][D], dtype, device, layer l at offset l*n_rows*D), per_layer[l] is layer
 * l's statistics (all of the same D). bf16 operands with D a multiple of 128 go to the tensor
 * cores in one launch per 48 layers, with the same tiles and the same reduction order as the
 * fused accumulation of ispa_attn_split: the results are identical bit for bit. */
int ispa_accum_ops(const ispa_stats *per_layer, int n_layers, const void *a_ops, const void *r_ops, int n_rows,
                   ispa_dtype dtype, ispa_stream_t stream);

/* 8-bit split attention [ISPA §3.4: the decomposition is built on 8-bit attention kernels,
 * SageAttention]: ispa_attn_split with S = scale * Q K^T taken from int8 copies of Q and K;
 * V, P, P V, the merge, the outputs and the fused statistics as in ispa_attn_split.
 * Quantisation (symmetric, float32, ties to even): s = amax / 127 and
 * x8 = clamp(rint(x * (127 / amax)), -127, 127), x8 = 0 and s = 0 where amax = 0; then
 * S_ij = scale * q_scale[i] * k_scale[block(j)] * (q8_i . k8_j), the dot product exact in int32.
 *
 * ispa_quantize_q_i8 -- q [n, heads, 128] bf16 -> q8 (same layout, int8), q_scale [n, heads]
 *   float32: one scale per (token, head). Device pointers; q, q8 16-byte aligned.
 * ispa_k_blocks -- number of K blocks of desc's layout (the size of a k_scale row): the KV
 *   rows cut at the partition boundaries into segments (the sink range, the chunk range and
 *   the history runs around them), each segment into blocks of 128 rows from its first row;
 *   blocks are numbered in row order. Returns the count (>= 0) or an error code.
 * ispa_quantize_k_i8 -- k [n_kv, heads, 128] bf16 -> k8 (same layout, int8), k_scale
 *   [heads, ispa_k_blocks(desc)] float32: one scale per (block, head).
 * ispa_attn_split_i8 -- as ispa_attn_split, with q8/q_scale and k8/k_scale from the two
 *   quantisers (k8 for the same desc) and v bf16. desc->dtype must be ISPA_BF16 and
 *   head_dim 128 (otherwise ISPA_ERR_UNSUPPORTED); the outputs are bf16. Workspace as for
 *   ispa_attn_split. */
int ispa_quantize_q_i8(const void *q, int n, int heads, int head_dim, signed char *q8, float *q_scale,
                       ispa_stream_t stream);
int ispa_k_blocks(const ispa_attn_desc *desc);
int ispa_quantize_k_i8(const ispa_attn_desc *desc, const void *k, signed char *k8, float *k_scale,
                       ispa_stream_t stream);
int ispa_attn_split_i8(const ispa_attn_desc *desc, const signed char *q8, const float *q_scale,
                       const signed char *k8, const float *k_scale, const void *v, void *o_full, float *lse_full,
                       void *o_loc, float *lse_loc, void *o_hist, float *lse_hist, const ispa_stats *stats,
                       void *ws, size_t ws_bytes, ispa_stream_t stream);

/* ispa_attn_split_noalloc -- ispa_attn_split with fused statistics for callers that cannot
 * allocate device memory (for example code running inside a host framework that owns all
 * device memory and passes only its inputs and outputs, or a plugin interface without a
 * workspace argument). The paper has no counterpart; this is a deployment variant. The
 * bf16 (or float32) operands handed from the attention kernel to the statistics GEMM live
 * in a static device array of 2 x 16 MiB instead of a caller workspace: each operand,
 * n_q * heads * head_dim elements, may take at most 16 MiB (8,388,608 bf16 or 4,194,304
 * float32 elements); larger calls return ISPA_ERR_UNSUPPORTED before any launch. stats is
 * required. The array is held by every GPU that loads the library until the process
 * exits. The first call on a device looks up the array's device address (make that first
 * call before any stream capture); the address is kept until the process exits, so a
 * cudaDeviceReset of that device ends the use of this call in the process. All calls share the array: calls that overlap on the
 * GPU race and must be serialised by the caller. Arguments otherwise as ispa_attn_split. */
int ispa_attn_split_noalloc(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                            void *o_full, float *lse_full, void *o_loc, float *lse_loc, void *o_hist,
                            float *lse_hist, const ispa_stats *stats, ispa_stream_t stream);

/* ispa_accum_stats -- the statistics of [ISPA §3.2] from attention outputs that were
 * computed elsewhere (unfused path): R = a_full - a_loc (then rounded to bf16 in bf16
 * mode), G += A_loc^T A_loc, C += A_loc^T R, H += R^T R, rows += n_rows.
 *   a_loc, a_full: [n_rows, D] device, dtype. ws: ispa_workspace_bytes(NULL, n_rows, D). */
int ispa_accum_stats(const ispa_stats *stats, const void *a_loc, const void *a_full, int n_rows,
                     ispa_dtype dtype, void *ws, size_t ws_bytes, ispa_stream_t stream);

/* ispa_stats_reset -- zero G, C, H and rows (start of a warmup, or a re-warmup after a
 * scene change [ISPA §3.1, §3.3]). */
int ispa_stats_reset(const ispa_stats *stats, ispa_stream_t stream);

/* ispa_solve_absorb -- Layer Absorb [ISPA §3.1 step 2, §3.2, §4.1 "Eq. 5"] and the
 * per-layer reconstruction error [ISPA §3.3], batched over layers:
 *   (G + lambda I) dW = C W, solved by a blocked Cholesky factorisation in float32;
 *   eps = E^2 / T^2 with E^2 = tr(dW^T G dW) - 2 tr(dW^T C W) + tr(W^T H W) and
 *   T^2 = tr(W^T (G + C + C^T + H) W) (relative squared error of the reconstructed
 *   projected output; eps = 0 when T^2 = 0).
 *   per_layer: host array of n_layers stats (device buffers, all with the same D).
 *   w_o: host array of n_layers device pointers to W [D, D] of w_dtype.
 *   dW: device [n_layers, D, D] float32.  eps: device [n_layers] float32.
 *   err_terms: optional device [n_layers, 2] double (E^2, T^2).
 *   w_new: optional host array of n_layers device pointers [D, D] w_dtype, written with
 *     W + dW (rounded to bf16 in bf16 mode) [ISPA §3.1 step 3].
 *   layer_status: device [n_layers] int, ISPA_OK or ISPA_ERR_NOT_SPD per layer (dW and
 *     eps of such a layer are NaN).
 *   ws: ispa_workspace_bytes(NULL, n_layers, D) bytes.
 * D must be a multiple of 64. With D a multiple of 128 every product runs on the tensor cores
 * (float32-accurate, 3xTF32) and the factorisation is blocked (512, 256 or 128 columns), the
 * diagonal blocks factored and inverted by thread-block clusters of 8 CTAs; otherwise the CUDA
 * cores do it all.
 * The layers run as up to three concurrent sub-batches, each in its own part of ws: the call
 * forks from `stream` onto two streams the library creates on its first call on a device
 * (driver objects, no device memory; make that first call before any stream capture) and joins
 * them back into `stream` with events, so the results are ordered on `stream` as for any other
 * call. Calls from several host threads are serialised while they enqueue. */
int ispa_solve_absorb(const ispa_stats *per_layer, int n_layers, const void *const *w_o,
                      ispa_dtype w_dtype, float lambda, float *dW, float *eps, double *err_terms,
                      void *const *w_new, int *layer_status, void *ws, size_t ws_bytes,
                      ispa_stream_t stream);

/* ispa_absorb_error -- the reconstruction error eps[l] of a GIVEN dW[l] on GIVEN statistics:
 * eps = E^2 / T^2 with E^2 = tr(dW^T G dW) - 2 tr(dW^T C W) + tr(W^T H W) and
 * T^2 = tr(W^T (G + C + C^T + H) W) [ISPA §3.3, the error the selection ranks; the same
 * formula ispa_solve_absorb evaluates after solving]. Without a solve it serves the
 * re-warmup trigger [ISPA §3.1 last paragraph, §3.3 last paragraph, which leave the
 * trigger open]: on the statistics of one chunk after the transition, eps of the dW solved
 * at the transition measures how well the absorbed projection still reconstructs the full
 * output of an F-layer.
 *   per_layer: n_layers statistics (device, as for ispa_solve_absorb); w_o, w_dtype: the
 *   original projections [D_in, D_out]; dW: n_layers device pointers to float32 [D][D]
 *   (16-byte aligned); eps: device float [n_layers]; err_terms: device double
 *   [n_layers][2] = (E^2, T^2), optional. eps = 0 when T^2 = 0.
 *   ws: ispa_workspace_bytes(NULL, n_layers, D) bytes (the solve's workspace suffices).
 * D must be a multiple of 64; the statistics are read only. */
int ispa_absorb_error(const ispa_stats *per_layer, int n_layers, const void *const *w_o,
                      ispa_dtype w_dtype, const float *const *dW, float *eps, double *err_terms,
                      void *ws, size_t ws_bytes, ispa_stream_t stream);

/* ispa_select_layers -- Dynamic Layer Selection [ISPA §3.3], host only: rank layers by
 * eps ascending (ties: lower layer index first; NaN last) and take the first K.
 *   eps_host [n_layers] (host), idx_out [min(K, n_layers)] (host, rank order),
 *   is_local [n_layers] (host, 1 for a selected layer), either output may be NULL. */
int ispa_select_layers(const float *eps_host, int n_layers, int K, int *idx_out,
                       unsigned char *is_local);

/* ispa_rewarm_check -- the re-warmup trigger's decision, host only [ISPA §3.1 last paragraph,
 * §3.3 last paragraph: the warmup is entered again when the scene changes; the pages give no
 * trigger. Reading: after a transition each monitored F-layer's live error -- ispa_absorb_error
 * of the transition's dW on one chunk's statistics -- is recorded per chunk; the warmup is
 * re-entered when a layer's latest live error exceeds both ratio x and min_rise + the lowest
 * live error that layer showed on the earlier chunks since the transition].
 *   live_history: host float [n_chunks][n_layers], oldest chunk first, NaN where a layer was not
 *     monitored in that chunk (an L-layer, or a layer the caller does not watch).
 *   ratio, min_rise: the rule's constants (the session uses 4 and 0.02); compared in double.
 *   fired: host [n_layers], set to 1 for a layer whose latest entry is a number, that has at least
 *     one earlier number, and whose latest value exceeds both bounds; 0 otherwise.
 * Returns the number of layers fired (>= 0), or an error code (nothing written). */
int ispa_rewarm_check(const float *live_history, int n_chunks, int n_layers, double ratio, double min_rise,
                      unsigned char *fired);

/* ispa_local_attn -- an L-layer after the switch [ISPA §3.1 step 3, §3.3]: attention
 * over the local rows only (every one of desc->n_kv rows of k_loc/v_loc, i.e. the sink
 * frame + current chunk; desc's range fields are ignored), and optionally the output
 * projection with the updated weights, y = O W_new.
 *   o [n_q, heads, head_dim] (device, dtype), lse [heads, n_q] (device, optional)
 *   w_new [D, D] (device, dtype, optional), y [n_q, D] (device, dtype; required iff
 *   w_new is given). ws: ispa_workspace_bytes(desc, 1, D) when w_new != NULL. */
int ispa_local_attn(const ispa_attn_desc *desc, const void *q, const void *k_loc,
                    const void *v_loc, void *o, float *lse, const void *w_new, void *y, void *ws,
                    size_t ws_bytes, ispa_stream_t stream);

/* ispa_project -- the attention output projection y = A W [ISPA §3.1 step 3: an L-layer's output
 * goes through the updated projection W_new = W + dW] on its own, the step that ispa_local_attn
 * runs after the attention when given w_new.
 *   a [n][d_in] (device, dtype; for an attention output [n, heads, head_dim] with d_in =
 *   heads*head_dim), w [d_in][d_out] (device, dtype), y [n][d_out] (device, dtype); all 16-byte
 *   aligned. bf16 with d_in and d_out multiples of 128 runs on the tensor cores (fp32
 *   accumulation, bf16 output); other shapes and float32 on the CUDA cores. */
int ispa_project(const void *a, int n, int d_in, const void *w, int d_out, void *y, ispa_dtype dtype,
                 ispa_stream_t stream);

/* ispa_quantize_w8 -- int8 weights for the W8A8 projection of the L-layers [ISPA §4.4: ISPA
 * is combined with 8-bit weights and activations; the scheme is not given -- reading:
 * symmetric int8, one scale per output column]. For each output column j of w [d_in][d_out]
 * (row-major, bf16 or float32, device): w_scale[j] = m / 127 with m = max_i |w[i][j]|, and
 * wq_t[j][i] = rint(w[i][j] * (127 / m)) clamped to [-127, 127] (float32 IEEE division and
 * multiplication, round to nearest even; a zero column gives scale 0 and codes 0). wq_t is
 * int8 [d_out][d_in] (transposed, 16-byte aligned), w_scale float32 [d_out]. d_in and d_out:
 * positive multiples of 128. Run once per transition on W_new. */
int ispa_quantize_w8(const void *w, ispa_dtype w_dtype, int d_in, int d_out, signed char *wq_t,
                     float *w_scale, ispa_stream_t stream);

/* ispa_project_w8a8 -- y = A W through int8 operands [ISPA §4.4, reading as for
 * ispa_quantize_w8]: each row r of a [n][d_in] (bf16, device, 16-byte aligned) is quantised
 * like a weight column (scale s_r = max|a_r| / 127), the int8 product accumulates exactly in
 * int32 on the tensor cores, and y[r][j] = bf16((float(acc) * s_r) * w_scale[j]) (round to
 * nearest even at each step) -- reproducible bit for bit. wq_t / w_scale from
 * ispa_quantize_w8; y [n][d_out] bf16 (device, 16-byte aligned). ws: scratch for the row codes
 * and scales, ispa_workspace_bytes(NULL, n, d_in) bytes (or the attention call's desc with
 * n_q = n). d_in and d_out: positive multiples of 128. */
int ispa_project_w8a8(const void *a, int n, int d_in, const signed char *wq_t, const float *w_scale,
                      int d_out, void *y, void *ws, size_t ws_bytes, ispa_stream_t stream);

/* ispa_workspace_bytes -- bytes of workspace that suffice for every call above with
 * these shapes: attention calls described by `desc` (may be NULL), ispa_accum_stats
 * and ispa_project_w8a8 with n rows of width D (when desc is NULL; with desc: n_q rows of
 * width heads*head_dim) and ispa_solve_absorb / ispa_absorb_error over n layers of size D. */
size_t ispa_workspace_bytes(const ispa_attn_desc *desc, int n, int D);

/* ispa_device_status -- synchronise `stream`, read and clear the current device's
 * error flag. Returns ISPA_OK, ISPA_ERR_TIMEOUT (a kernel's bounded wait ran out and the
 * kernel returned early; its outputs are not valid) or ISPA_ERR_CUDA. */
int ispa_device_status(ispa_stream_t stream);

/* ispa_selftest_bounded_wait -- test hook for the failure path: launches one kernel that
 * waits on an mbarrier nothing ever arrives on, with a limit of `limit_us` microseconds
 * (1..1000000), after which the kernel records ISPA_ERR_TIMEOUT in the device flag and
 * returns. The GPU context stays usable. */
int ispa_selftest_bounded_wait(unsigned limit_us, ispa_stream_t stream);

/* ispa_selftest_exp2_poly -- test hook: y[i] = 2^x[i] computed by the FMA-pipe
 * exponential the split-attention softmax uses for part of its weights (range reduction
 * + degree-3 polynomial): elements 2q, 2q+1 by its packed two-lane form, an odd last
 * element by its scalar form. x, y: device float32 [n]. Valid for x <= 64; x < -125 gives
 * a value below 3e-38. */
int ispa_selftest_exp2_poly(const float *x, float *y, int n, ispa_stream_t stream);

/* ispa_set_attn_kernel -- choose the tensor-core kernel that bf16 attention calls with
 * head_dim 128 use (ispa_attn_split, ispa_attn_split_noalloc, ispa_local_attn), for this
 * process and every device. All compute the same result:
 *   ISPA_ATTN_AUTO (0)      the fastest one on sm_100a: the two-group kernel (on a 1.3B
 *                           layer call 13 % faster than the single-group one, which is
 *                           1.8x faster than the pair kernel);
 *   ISPA_ATTN_SINGLE (1)    one CTA per 128-query tile, one softmax group, all MMAs
 *                           cta_group::1;
 *   ISPA_ATTN_PAIR (2)      two CTAs (a cluster of 2 on two SMs) per pair of 128-query
 *                           tiles of one head: 256-row cta_group::2 MMAs, each SM loading
 *                           half of every K/V tile;
 *   ISPA_ATTN_TWO_GROUP (3) one CTA per 128-query tile with two softmax groups that take
 *                           alternate KV tiles, each with its own S buffer and accumulator
 *                           in tensor memory, merged by log-sum-exp at the end.
 * head_dim 64 always uses the single-group kernel. Returns the previous choice, or
 * ISPA_ERR_INVALID_ARG (nothing changed) for any other value. Not synchronised with
 * launches in flight: set it before the calls it should affect. */
typedef enum {
    ISPA_ATTN_AUTO = 0,
    ISPA_ATTN_SINGLE = 1,
    ISPA_ATTN_PAIR = 2,
    ISPA_ATTN_TWO_GROUP = 3
} ispa_attn_kernel;
int ispa_set_attn_kernel(int choice);

/* ispa_kernel_launches -- number of kernels this library has launched in this process
 * (every device, every stream), for accounting; never reset. */
unsigned long long ispa_kernel_launches(void);

/* ispa_last_error -- message of the last failing call on this host thread ("" if none). */
const char *ispa_last_error(void);

/* ispa_version -- library version string. */
const char *ispa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ISPA_H */
