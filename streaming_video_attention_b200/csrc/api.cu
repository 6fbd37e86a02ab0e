// C-ABI entry points of libispa: argument checks, workspace layout and dispatch to the
// kernels. Every call enqueues on the caller's stream and allocates nothing.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
cudaError_t error_batch(const PtrBatch &G, const PtrBatch &C, const PtrBatch &H, const PtrBatch &W, ElemType wt,
                        const PtrBatch &dW, const PtrBatch &Y, const PtrBatch &P, float *Yc, float *Pc, float *split,
                        double *terms, int nparts, float *eps, double *err_terms, int D, int batch, int *err_flag,
                        cudaStream_t s);
cudaError_t solve_batch(const PtrBatch &G, const PtrBatch &C, const PtrBatch &H, const PtrBatch &W, ElemType wt,
                        const PtrBatch &dW, const PtrBatch &M, const PtrBatch &Y, const PtrBatch &P, float *Yc,
                        float *Pc, float *split, double *terms, int nparts, int *status, float *eps,
                        double *err_terms, const PtrBatch *w_new, int D, float lambda, int batch, int *err_flag,
                        cudaStream_t s);
}

namespace ispa {
static std::atomic<unsigned long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
int record_error(int code, const char *msg);
}  // namespace ispa

using namespace ispa;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *where) {
    return fail(ISPA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

}  // namespace

// Lets entry points defined in other files report through ispa_last_error().
int ispa::record_error(int code, const char *msg) { return fail(code, "%s", msg); }

namespace {

#define CUDA_CHECK_RET(x, where)                     \
    do {                                             \
        cudaError_t e_ = (x);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// Per-device error flag, shared by every kernel of the library. Host code never touches
// the symbol directly: its device address is looked up once per device.
__device__ int g_device_error_flag;

constexpr int kMaxDevices = 64;
std::mutex g_flag_mutex;
int *g_flag_ptr[kMaxDevices] = {nullptr};

int device_error_flag(int **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(ISPA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_flag_mutex);
    if (!g_flag_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error_flag);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error flag)");
        g_flag_ptr[dev] = static_cast<int *>(p);
    }
    *out = g_flag_ptr[dev];
    return ISPA_OK;
}

// Streams and events that let a batched solve run its layers as several concurrent sub-batches:
// the Cholesky and triangular-solve chain of one sub-batch is a sequence of small, latency-bound
// kernels, and the large products of another fill the SMs meanwhile. Created once per device
// (driver objects, no device memory) and reused; calls that use them are serialised on the host.
constexpr int kSolveStreams = 3;
struct SideStreams {
    cudaStream_t st[kSolveStreams - 1];
    cudaEvent_t fork, join[kSolveStreams - 1];
    bool ready;
};
std::mutex g_side_mutex;
SideStreams g_side[kMaxDevices];

int side_streams(SideStreams **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(ISPA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    SideStreams &ss = g_side[dev];
    if (!ss.ready) {
        for (int i = 0; i < kSolveStreams - 1; ++i) {
            e = cudaStreamCreateWithFlags(&ss.st[i], cudaStreamNonBlocking);
            if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
            e = cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming);
            if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreateWithFlags");
        }
        e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreateWithFlags");
        ss.ready = true;
    }
    *out = &ss;
    return ISPA_OK;
}

size_t elem_size(ispa_dtype t) { return t == ISPA_BF16 ? 2 : 4; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace of one attention call with fused statistics: A_loc and R operands.
size_t attn_ws_bytes(const ispa_attn_desc *d) {
    const size_t D = (size_t)d->heads * d->head_dim;
    return 2 * align_up((size_t)d->n_q * D * elem_size(d->dtype), 256);
}

size_t accum_ws_bytes(int n_rows, int D, ispa_dtype t) {
    return align_up((size_t)n_rows * D * elem_size(t), 256);
}

// ispa_project_w8a8: int8 codes [n][D] then float scales [n]
size_t w8a8_ws_bytes(int n_rows, int D) {
    return align_up((size_t)n_rows * D, 256) + align_up((size_t)n_rows * sizeof(float), 256);
}

// Partial sums per layer and trace of the reconstruction error: with D a multiple of 128 the D x D
// products run on the tensor cores and every 128 x 128 output tile contributes one partial from
// its epilogue; otherwise a reduction kernel writes 64.
int eps_parts(int D) { return D % 128 == 0 ? (D / 128) * (D / 128) : 64; }

size_t solve_ws_bytes(int n_layers, int D) {
    const size_t b = (size_t)std::min(n_layers, kMaxBatch);
    const size_t mat = (size_t)D * D * sizeof(float);   // D is a multiple of 64: 256-byte multiple
    return b * 9 * mat + align_up(5 * b * (size_t)eps_parts(D) * sizeof(double), 256);
}

int check_desc(const ispa_attn_desc *d, bool need_ranges) {
    if (!d) return fail(ISPA_ERR_INVALID_ARG, "desc is NULL");
    if (d->n_q < 0 || d->n_kv < 0 || d->heads <= 0) return fail(ISPA_ERR_INVALID_ARG, "bad sizes n_q=%d n_kv=%d heads=%d", d->n_q, d->n_kv, d->heads);
    if (d->head_dim != 64 && d->head_dim != 128) return fail(ISPA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", d->head_dim);
    if (d->dtype != ISPA_BF16 && d->dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad dtype %d", (int)d->dtype);
    if (!(d->scale > 0.f) || !(d->scale < 1e30f)) return fail(ISPA_ERR_INVALID_ARG, "bad scale");
    if ((long long)d->n_kv * d->heads * d->head_dim >= (1ll << 40)) return fail(ISPA_ERR_UNSUPPORTED, "KV too large");
    if (need_ranges) {
        auto okr = [&](int b, int e) { return 0 <= b && b <= e && e <= d->n_kv; };
        if (!okr(d->sink_begin, d->sink_end)) return fail(ISPA_ERR_INVALID_ARG, "sink range [%d,%d) outside [0,%d)", d->sink_begin, d->sink_end, d->n_kv);
        if (!okr(d->chunk_begin, d->chunk_end)) return fail(ISPA_ERR_INVALID_ARG, "chunk range [%d,%d) outside [0,%d)", d->chunk_begin, d->chunk_end, d->n_kv);
        const bool se = d->sink_begin == d->sink_end, ce = d->chunk_begin == d->chunk_end;
        if (!se && !ce && d->sink_begin < d->chunk_end && d->chunk_begin < d->sink_end)
            return fail(ISPA_ERR_INVALID_ARG, "sink and chunk ranges overlap");
    }
    return ISPA_OK;
}

// Local segments first (in row order), then the history gaps.
SegmentList make_segments(const ispa_attn_desc *d, bool local_only) {
    SegmentList L;
    L.count = 0;
    if (local_only) {
        if (d->n_kv > 0) L.seg[L.count++] = {0, d->n_kv, 0};
        return L;
    }
    std::vector<std::pair<int, int>> loc;
    if (d->sink_end > d->sink_begin) loc.push_back({d->sink_begin, d->sink_end});
    if (d->chunk_end > d->chunk_begin) loc.push_back({d->chunk_begin, d->chunk_end});
    std::sort(loc.begin(), loc.end());
    for (auto &r : loc) L.seg[L.count++] = {r.first, r.second, 0};
    int cur = 0;
    for (auto &r : loc) {
        if (r.first > cur) L.seg[L.count++] = {cur, r.first, 1};
        cur = std::max(cur, r.second);
    }
    if (cur < d->n_kv) L.seg[L.count++] = {cur, d->n_kv, 1};
    return L;
}

__global__ void add_rows_kernel(long long *rows, long long n) { *rows += n; }

struct RowsBatch {
    long long *r[kMaxBatch];
};
__global__ void add_rows_batch_kernel(RowsBatch rows, int layers, long long n) {
    if (threadIdx.x < layers) *rows.r[threadIdx.x] += n;
}

template <typename T>
__global__ void residual_kernel(const T *a_loc, const T *a_full, T *r, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        r[i] = from_f32<T>(to_f32(a_full[i]) - to_f32(a_loc[i]));
}

// G += A^T A, C += A^T R, H += R^T R, rows += n, for operands [n, D] of type t.
int accumulate(const ispa_stats *st, const void *a_ops, const void *r_ops, int n, ispa_dtype t, int *flag,
               cudaStream_t s) {
    const int D = st->D;
    if (n > 0) {
        if (t == ISPA_BF16) {
            CUDA_CHECK_RET(launch_stats_bf16(a_ops, r_ops, n, D, st->G, st->C, st->H, flag, s), "stats GEMM (bf16)");
        } else {
            const ElemType et = ElemType::F32;
            GemmDesc g{D, D, n, D, D, D, false, false, et, et, ElemType::F32, 1.f, 1.f, false, 1};
            GemmBatch b;
            b.A[0] = a_ops; b.B[0] = a_ops; b.C[0] = st->G;
            CUDA_CHECK_RET(launch_gemm_simt(g, b, s), "stats GEMM G");
            b.A[0] = a_ops; b.B[0] = r_ops; b.C[0] = st->C;
            CUDA_CHECK_RET(launch_gemm_simt(g, b, s), "stats GEMM C");
            b.A[0] = r_ops; b.B[0] = r_ops; b.C[0] = st->H;
            CUDA_CHECK_RET(launch_gemm_simt(g, b, s), "stats GEMM H");
        }
    }
    add_rows_kernel<<<1, 1, 0, s>>>(st->rows, n); note_launch();
    CUDA_CHECK_RET(cudaGetLastError(), "rows counter");
    return ISPA_OK;
}

int check_stats(const ispa_stats *st, int D) {
    if (!st) return fail(ISPA_ERR_INVALID_ARG, "stats is NULL");
    if (st->D != D) return fail(ISPA_ERR_INVALID_ARG, "stats D=%d but the attention has D=%d", st->D, D);
    if (!st->G || !st->C || !st->H || !st->rows) return fail(ISPA_ERR_INVALID_ARG, "stats has a NULL buffer");
    if (!aligned(st->G, 16) || !aligned(st->C, 16) || !aligned(st->H, 16)) return fail(ISPA_ERR_INVALID_ARG, "stats buffers must be 16-byte aligned");
    return ISPA_OK;
}

int check_ws(void *ws, size_t have, size_t need) {
    if (need == 0) return ISPA_OK;
    if (!ws) return fail(ISPA_ERR_WORKSPACE, "workspace of %zu bytes required, got NULL", need);
    if (!aligned(ws, 256)) return fail(ISPA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (have < need) return fail(ISPA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", have, need);
    return ISPA_OK;
}

// Kernel used by bf16 head_dim-128 attention (ispa_set_attn_kernel).
std::atomic<int> g_attn_kernel{ISPA_ATTN_AUTO};

// q_scale / k_scale non-null: q and k are int8 (the 8-bit split attention).
int run_attention(const ispa_attn_desc *d, const void *q, const void *k, const void *v, void *o_full, float *lse_full,
                  void *o_loc, float *lse_loc, void *o_hist, float *lse_hist, void *a_ops, void *r_ops,
                  bool local_only, cudaStream_t s, const float *q_scale = nullptr, const float *k_scale = nullptr) {
    int *flag = nullptr;
    int rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    AttnArgs a;
    a.q = q; a.k = k; a.v = v;
    a.o_full = o_full; a.lse_full = lse_full;
    a.o_loc = o_loc; a.lse_loc = lse_loc;
    a.o_hist = o_hist; a.lse_hist = lse_hist;
    a.a_loc_ops = a_ops; a.r_ops = r_ops;
    a.n_q = d->n_q; a.n_kv = d->n_kv; a.heads = d->heads; a.head_dim = d->head_dim;
    a.scale = d->scale;
    a.segs = make_segments(d, local_only);
    a.err_flag = flag;
    cudaError_t e;
    if (q_scale)
        e = launch_attn_i8_2g(a, q_scale, k_scale, s);
    else if (d->dtype == ISPA_FP32)
        e = launch_attn_simt_f32(a, s);
    else if (d->head_dim != 128)
        e = launch_attn_bf16(a, s);
    else {
        const int choice = g_attn_kernel.load(std::memory_order_relaxed);
        if (choice == ISPA_ATTN_PAIR)
            e = launch_attn_bf16_2sm(a, s);
        else if (choice == ISPA_ATTN_SINGLE)
            e = launch_attn_bf16(a, s);
        else
            e = launch_attn_bf16_2g(a, s);   // ISPA_ATTN_AUTO, ISPA_ATTN_TWO_GROUP
    }
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
    return ISPA_OK;
}

__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int *flag) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing ever arrives on `bar`: the wait must run out and record the timeout.
        ptx::mbar_wait_bounded(&bar, 0, limit_ns, flag, nullptr);
    }
    __syncthreads();
}

// Pairs (2q, 2q+1) through the packed form the softmax uses; an odd last element through the
// scalar form.
__global__ void exp2_poly_selftest_kernel(const float *x, float *y, int n) {
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; 2 * q < n; q += gridDim.x * blockDim.x) {
        if (2 * q + 1 < n) {
            const uint64_t r = ptx::exp2_poly2(ptx::f2_pack(x[2 * q], x[2 * q + 1]));
            y[2 * q] = ptx::f2_lo(r);
            y[2 * q + 1] = ptx::f2_hi(r);
        } else {
            y[2 * q] = ptx::exp2_poly(x[2 * q]);
        }
    }
}

}  // namespace

extern "C" {

int ispa_selftest_exp2_poly(const float *x, float *y, int n, ispa_stream_t stream) {
    g_last_error.clear();
    if (n < 0 || (n > 0 && (!x || !y))) return fail(ISPA_ERR_INVALID_ARG, "bad arguments");
    if (n == 0) return ISPA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    exp2_poly_selftest_kernel<<<std::min((n + 255) / 256, 1024), 256, 0, s>>>(x, y, n);
    note_launch();
    CUDA_CHECK_RET(cudaGetLastError(), "selftest launch");
    return ISPA_OK;
}

const char *ispa_last_error(void) { return g_last_error.c_str(); }

unsigned long long ispa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char *ispa_version(void) { return "ispa-b200 0.1 (sm_100a)"; }

size_t ispa_workspace_bytes(const ispa_attn_desc *desc, int n, int D) {
    size_t need = 0;
    if (desc) {
        need = std::max(need, attn_ws_bytes(desc));
        const size_t Dd = (size_t)desc->heads * desc->head_dim;
        need = std::max(need, align_up((size_t)desc->n_q * Dd * elem_size(desc->dtype), 256));
        need = std::max(need, w8a8_ws_bytes(desc->n_q, (int)Dd));
    } else if (n > 0 && D > 0) {
        need = std::max(need, accum_ws_bytes(n, D, ISPA_FP32));
        need = std::max(need, w8a8_ws_bytes(n, D));
    }
    if (n > 0 && D > 0) need = std::max(need, solve_ws_bytes(n, D));
    return need;
}

static int attn_split_impl(const ispa_attn_desc *desc, const void *q, const void *k, const void *v, void *o_full,
                           float *lse_full, void *o_loc, float *lse_loc, void *o_hist, float *lse_hist,
                           const ispa_stats *stats, void *ws, size_t ws_bytes, ispa_stream_t stream,
                           const float *q_scale, const float *k_scale) {
    int rc;
    if (desc->n_q > 0 && (!q || !o_full || !lse_full)) return fail(ISPA_ERR_INVALID_ARG, "q, o_full and lse_full are required");
    if (desc->n_kv > 0 && (!k || !v)) return fail(ISPA_ERR_INVALID_ARG, "k and v are required");
    for (const void *p : {q, k, v, (const void *)o_full, (const void *)o_loc, (const void *)o_hist})
        if (p && !aligned(p, 16)) return fail(ISPA_ERR_INVALID_ARG, "q/k/v/o buffers must be 16-byte aligned");
    const int D = desc->heads * desc->head_dim;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *a_ops = nullptr, *r_ops = nullptr;
    if (stats) {
        rc = check_stats(stats, D);
        if (rc != ISPA_OK) return rc;
        rc = check_ws(ws, ws_bytes, attn_ws_bytes(desc));
        if (rc != ISPA_OK) return rc;
        a_ops = ws;
        r_ops = static_cast<char *>(ws) + align_up((size_t)desc->n_q * D * elem_size(desc->dtype), 256);
    }
    if (desc->n_q > 0) {
        rc = run_attention(desc, q, k, v, o_full, lse_full, o_loc, lse_loc, o_hist, lse_hist, a_ops, r_ops, false, s,
                           q_scale, k_scale);
        if (rc != ISPA_OK) return rc;
    }
    if (stats) {
        int *flag = nullptr;
        rc = device_error_flag(&flag);
        if (rc != ISPA_OK) return rc;
        return accumulate(stats, a_ops, r_ops, desc->n_q, desc->dtype, flag, s);
    }
    return ISPA_OK;
}

int ispa_attn_split(const ispa_attn_desc *desc, const void *q, const void *k, const void *v, void *o_full,
                    float *lse_full, void *o_loc, float *lse_loc, void *o_hist, float *lse_hist,
                    const ispa_stats *stats, void *ws, size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    int rc = check_desc(desc, true);
    if (rc != ISPA_OK) return rc;
    return attn_split_impl(desc, q, k, v, o_full, lse_full, o_loc, lse_loc, o_hist, lse_hist, stats, ws, ws_bytes,
                           stream, nullptr, nullptr);
}

int ispa_attn_split_ops(const ispa_attn_desc *desc, const void *q, const void *k, const void *v, void *o_full,
                        float *lse_full, void *o_loc, float *lse_loc, void *o_hist, float *lse_hist, void *a_ops,
                        void *r_ops, ispa_stream_t stream) {
    g_last_error.clear();
    int rc = check_desc(desc, true);
    if (rc != ISPA_OK) return rc;
    if (desc->n_q > 0 && (!a_ops || !r_ops)) return fail(ISPA_ERR_INVALID_ARG, "a_ops and r_ops are required");
    if ((a_ops && !aligned(a_ops, 16)) || (r_ops && !aligned(r_ops, 16)))
        return fail(ISPA_ERR_INVALID_ARG, "a_ops and r_ops must be 16-byte aligned");
    if (desc->n_q > 0 && (!q || !o_full || !lse_full)) return fail(ISPA_ERR_INVALID_ARG, "q, o_full and lse_full are required");
    if (desc->n_kv > 0 && (!k || !v)) return fail(ISPA_ERR_INVALID_ARG, "k and v are required");
    for (const void *p : {q, k, v, (const void *)o_full, (const void *)o_loc, (const void *)o_hist})
        if (p && !aligned(p, 16)) return fail(ISPA_ERR_INVALID_ARG, "q/k/v/o buffers must be 16-byte aligned");
    if (desc->n_q == 0) return ISPA_OK;
    return run_attention(desc, q, k, v, o_full, lse_full, o_loc, lse_loc, o_hist, lse_hist, a_ops, r_ops, false,
                         reinterpret_cast<cudaStream_t>(stream));
}

int ispa_accum_ops(const ispa_stats *per_layer, int n_layers, const void *a_ops, const void *r_ops, int n_rows,
                   ispa_dtype dtype, ispa_stream_t stream) {
    g_last_error.clear();
    if (!per_layer || n_layers < 0) return fail(ISPA_ERR_INVALID_ARG, "per_layer is NULL or n_layers < 0");
    if (dtype != ISPA_BF16 && dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad dtype");
    if (n_rows < 0) return fail(ISPA_ERR_INVALID_ARG, "n_rows < 0");
    if (n_layers == 0) return ISPA_OK;
    const int D = per_layer[0].D;
    if (D <= 0) return fail(ISPA_ERR_INVALID_ARG, "D <= 0");
    for (int l = 0; l < n_layers; ++l) {
        int rc = check_stats(&per_layer[l], D);
        if (rc != ISPA_OK) return fail(rc, "layer %d: %s", l, g_last_error.c_str());
    }
    if (n_rows > 0 && (!a_ops || !r_ops)) return fail(ISPA_ERR_INVALID_ARG, "a_ops and r_ops are required");
    if ((a_ops && !aligned(a_ops, 16)) || (r_ops && !aligned(r_ops, 16)))
        return fail(ISPA_ERR_INVALID_ARG, "a_ops and r_ops must be 16-byte aligned");
    if (dtype == ISPA_BF16 && D % 64 != 0) return fail(ISPA_ERR_UNSUPPORTED, "bf16 statistics need D %% 64 == 0");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int *flag = nullptr;
    int rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    const size_t per = (size_t)n_rows * D * elem_size(dtype);
    for (int l0 = 0; l0 < n_layers; l0 += kMaxBatch) {
        const int b = std::min(kMaxBatch, n_layers - l0);
        const char *a = static_cast<const char *>(a_ops) + (size_t)l0 * per;
        const char *r = static_cast<const char *>(r_ops) + (size_t)l0 * per;
        if (dtype == ISPA_BF16 && n_rows > 0) {
            float *G[kMaxBatch], *C[kMaxBatch], *H[kMaxBatch];
            for (int z = 0; z < b; ++z) {
                G[z] = per_layer[l0 + z].G; C[z] = per_layer[l0 + z].C; H[z] = per_layer[l0 + z].H;
            }
            CUDA_CHECK_RET(launch_stats_bf16_layers(a, r, b, n_rows, D, G, C, H, flag, s), "stats GEMM (bf16, layers)");
            RowsBatch rows;
            for (int z = 0; z < b; ++z) rows.r[z] = per_layer[l0 + z].rows;
            add_rows_batch_kernel<<<1, 64, 0, s>>>(rows, b, n_rows); note_launch();
            CUDA_CHECK_RET(cudaGetLastError(), "rows counters");
        } else {
            for (int z = 0; z < b; ++z) {
                rc = accumulate(&per_layer[l0 + z], a + (size_t)z * per, r + (size_t)z * per, n_rows, dtype, flag, s);
                if (rc != ISPA_OK) return rc;
            }
        }
    }
    return ISPA_OK;
}

// K blocks of the 8-bit split attention: the KV segments in row order, each cut into
// blocks of 128 rows from its first row.
static SegmentList row_order_segments(const ispa_attn_desc *d) {
    SegmentList L = make_segments(d, false);
    std::sort(L.seg, L.seg + L.count, [](const Segment &a, const Segment &b) { return a.begin < b.begin; });
    return L;
}

static int count_k_blocks(const ispa_attn_desc *d) {
    const SegmentList L = row_order_segments(d);
    int n = 0;
    for (int i = 0; i < L.count; ++i) n += (L.seg[i].end - L.seg[i].begin + 127) / 128;
    return n;
}

static int check_i8_desc(const ispa_attn_desc *desc) {
    int rc = check_desc(desc, true);
    if (rc != ISPA_OK) return rc;
    if (desc->dtype != ISPA_BF16 || desc->head_dim != 128)
        return fail(ISPA_ERR_UNSUPPORTED, "8-bit split attention: bf16 V and outputs, head_dim 128 only");
    return ISPA_OK;
}

int ispa_k_blocks(const ispa_attn_desc *desc) {
    g_last_error.clear();
    int rc = check_desc(desc, true);
    if (rc != ISPA_OK) return rc;
    return count_k_blocks(desc);
}

int ispa_quantize_q_i8(const void *q, int n, int heads, int head_dim, signed char *q8, float *q_scale,
                       ispa_stream_t stream) {
    g_last_error.clear();
    if (n < 0 || heads <= 0) return fail(ISPA_ERR_INVALID_ARG, "bad sizes n=%d heads=%d", n, heads);
    if (head_dim != 128) return fail(ISPA_ERR_UNSUPPORTED, "head_dim %d (supported: 128)", head_dim);
    if (n == 0) return ISPA_OK;
    if (!q || !q8 || !q_scale) return fail(ISPA_ERR_INVALID_ARG, "q, q8 and q_scale are required");
    if (!aligned(q, 16) || !aligned(q8, 16)) return fail(ISPA_ERR_INVALID_ARG, "q and q8 must be 16-byte aligned");
    cudaError_t e = launch_quant_q_i8(q, n, heads, reinterpret_cast<int8_t *>(q8), q_scale,
                                      reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quantize q");
    return ISPA_OK;
}

int ispa_quantize_k_i8(const ispa_attn_desc *desc, const void *k, signed char *k8, float *k_scale,
                       ispa_stream_t stream) {
    g_last_error.clear();
    int rc = check_i8_desc(desc);
    if (rc != ISPA_OK) return rc;
    if (desc->n_kv == 0) return ISPA_OK;
    if (!k || !k8 || !k_scale) return fail(ISPA_ERR_INVALID_ARG, "k, k8 and k_scale are required");
    if (!aligned(k, 16) || !aligned(k8, 16)) return fail(ISPA_ERR_INVALID_ARG, "k and k8 must be 16-byte aligned");
    cudaError_t e = launch_quant_k_i8(k, desc->heads, row_order_segments(desc), count_k_blocks(desc),
                                      reinterpret_cast<int8_t *>(k8), k_scale, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quantize k");
    return ISPA_OK;
}

int ispa_attn_split_i8(const ispa_attn_desc *desc, const signed char *q8, const float *q_scale,
                       const signed char *k8, const float *k_scale, const void *v, void *o_full, float *lse_full,
                       void *o_loc, float *lse_loc, void *o_hist, float *lse_hist, const ispa_stats *stats, void *ws,
                       size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    int rc = check_i8_desc(desc);
    if (rc != ISPA_OK) return rc;
    if (desc->n_q > 0 && !q_scale) return fail(ISPA_ERR_INVALID_ARG, "q_scale is required");
    if (desc->n_kv > 0 && !k_scale) return fail(ISPA_ERR_INVALID_ARG, "k_scale is required");
    return attn_split_impl(desc, q8, k8, v, o_full, lse_full, o_loc, lse_loc, o_hist, lse_hist, stats, ws, ws_bytes,
                           stream, q_scale, k_scale);
}

int ispa_accum_stats(const ispa_stats *stats, const void *a_loc, const void *a_full, int n_rows, ispa_dtype dtype,
                     void *ws, size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    if (!stats) return fail(ISPA_ERR_INVALID_ARG, "stats is NULL");
    if (dtype != ISPA_BF16 && dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad dtype");
    if (n_rows < 0) return fail(ISPA_ERR_INVALID_ARG, "n_rows < 0");
    int rc = check_stats(stats, stats->D);
    if (rc != ISPA_OK) return rc;
    if (stats->D <= 0) return fail(ISPA_ERR_INVALID_ARG, "D <= 0");
    if (n_rows > 0 && (!a_loc || !a_full)) return fail(ISPA_ERR_INVALID_ARG, "a_loc and a_full are required");
    if ((a_loc && !aligned(a_loc, 16)) || (a_full && !aligned(a_full, 16))) return fail(ISPA_ERR_INVALID_ARG, "a_loc/a_full must be 16-byte aligned");
    if (dtype == ISPA_BF16 && stats->D % 64 != 0) return fail(ISPA_ERR_UNSUPPORTED, "bf16 statistics need D %% 64 == 0");
    rc = check_ws(ws, ws_bytes, n_rows > 0 ? accum_ws_bytes(n_rows, stats->D, dtype) : 0);
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int *flag = nullptr;
    rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    const size_t n = (size_t)n_rows * stats->D;
    if (n > 0) {
        const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
        if (dtype == ISPA_BF16)
            residual_kernel<bf16><<<blocks, 256, 0, s>>>((const bf16 *)a_loc, (const bf16 *)a_full, (bf16 *)ws, n);
        else
            residual_kernel<float><<<blocks, 256, 0, s>>>((const float *)a_loc, (const float *)a_full, (float *)ws, n);
        note_launch();
        CUDA_CHECK_RET(cudaGetLastError(), "residual kernel");
    }
    return accumulate(stats, a_loc, ws, n_rows, dtype, flag, s);
}

int ispa_stats_reset(const ispa_stats *stats, ispa_stream_t stream) {
    g_last_error.clear();
    if (!stats) return fail(ISPA_ERR_INVALID_ARG, "stats is NULL");
    int rc = check_stats(stats, stats->D);
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t b = (size_t)stats->D * stats->D * sizeof(float);
    CUDA_CHECK_RET(cudaMemsetAsync(stats->G, 0, b, s), "memset G");
    CUDA_CHECK_RET(cudaMemsetAsync(stats->C, 0, b, s), "memset C");
    CUDA_CHECK_RET(cudaMemsetAsync(stats->H, 0, b, s), "memset H");
    CUDA_CHECK_RET(cudaMemsetAsync(stats->rows, 0, sizeof(long long), s), "memset rows");
    return ISPA_OK;
}

int ispa_solve_absorb(const ispa_stats *per_layer, int n_layers, const void *const *w_o, ispa_dtype w_dtype,
                      float lambda, float *dW, float *eps, double *err_terms, void *const *w_new, int *layer_status,
                      void *ws, size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    if (n_layers < 0) return fail(ISPA_ERR_INVALID_ARG, "n_layers < 0");
    if (n_layers == 0) return ISPA_OK;
    if (!per_layer || !w_o || !dW || !eps || !layer_status) return fail(ISPA_ERR_INVALID_ARG, "per_layer, w_o, dW, eps and layer_status are required");
    if (w_dtype != ISPA_BF16 && w_dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad w_dtype");
    if (!(lambda >= 0.f) || !(lambda < 1e30f)) return fail(ISPA_ERR_INVALID_ARG, "lambda must be finite and >= 0");
    const int D = per_layer[0].D;
    if (D <= 0 || D % 64 != 0) return fail(ISPA_ERR_UNSUPPORTED, "D=%d: the solve needs D %% 64 == 0", D);
    for (int l = 0; l < n_layers; ++l) {
        int rc = check_stats(&per_layer[l], D);
        if (rc != ISPA_OK) return fail(rc, "layer %d: %s", l, g_last_error.c_str());
        if (!w_o[l]) return fail(ISPA_ERR_INVALID_ARG, "w_o[%d] is NULL", l);
        if (w_new && !w_new[l]) return fail(ISPA_ERR_INVALID_ARG, "w_new[%d] is NULL", l);
    }
    if (!aligned(dW, 16)) return fail(ISPA_ERR_INVALID_ARG, "dW must be 16-byte aligned");
    int rc = check_ws(ws, ws_bytes, solve_ws_bytes(n_layers, D));
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    CUDA_CHECK_RET(cudaMemsetAsync(layer_status, 0, sizeof(int) * n_layers, s), "memset layer_status");

    // workspace: M, Y, P blocks of bmax D x D float32 matrices each (contiguous per block), the
    // 3xTF32 split operands (6 blocks), then the trace partial sums
    const size_t mat = (size_t)D * D * sizeof(float);
    const int bmax = std::min(n_layers, kMaxBatch);
    char *wsb = static_cast<char *>(ws);
    char *Mb = wsb, *Yb = wsb + (size_t)bmax * mat, *Pb = wsb + 2 * (size_t)bmax * mat;
    float *split = reinterpret_cast<float *>(wsb + 3 * (size_t)bmax * mat);
    double *terms = reinterpret_cast<double *>(wsb + 9 * (size_t)bmax * mat);
    int *flag = nullptr;
    rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    // Each chunk of up to kMaxBatch layers runs as up to kSolveStreams concurrent sub-batches: the
    // first on `stream`, the others on side streams forked from and joined back into it. Every
    // sub-batch uses its own slices of the workspace (its layers' M, Y, P and split blocks, its
    // trace sums).
    SideStreams *side = nullptr;
    std::unique_lock<std::mutex> side_lock(g_side_mutex, std::defer_lock);
    const int max_sub = std::min(kSolveStreams, n_layers);
    if (max_sub > 1) {
        side_lock.lock();
        rc = side_streams(&side);
        if (rc != ISPA_OK) return rc;
    }
    const size_t nD = (size_t)D * D;
    for (int l0 = 0; l0 < n_layers; l0 += kMaxBatch) {
        const int b = std::min(kMaxBatch, n_layers - l0);
        const int nsub = std::min(max_sub, b);
        if (nsub > 1) {
            CUDA_CHECK_RET(cudaEventRecord(side->fork, s), "cudaEventRecord (fork)");
            for (int i = 0; i < nsub - 1; ++i)
                CUDA_CHECK_RET(cudaStreamWaitEvent(side->st[i], side->fork, 0), "cudaStreamWaitEvent (fork)");
        }
        for (int sb = 0; sb < nsub; ++sb) {
            const int z0 = b * sb / nsub, z1 = b * (sb + 1) / nsub, bs = z1 - z0;
            cudaStream_t ss = sb == 0 ? s : side->st[sb - 1];
            PtrBatch G, C, H, W, DW, M, Y, P, WN;
            for (int z = 0; z < bs; ++z) {
                const int l = l0 + z0 + z;
                const ispa_stats &st = per_layer[l];
                G.p[z] = st.G; C.p[z] = st.C; H.p[z] = st.H;
                W.p[z] = const_cast<void *>(w_o[l]);
                DW.p[z] = dW + (size_t)l * nD;
                M.p[z] = Mb + (size_t)(z0 + z) * mat;
                Y.p[z] = Yb + (size_t)(z0 + z) * mat;
                P.p[z] = Pb + (size_t)(z0 + z) * mat;
                if (w_new) WN.p[z] = w_new[l];
            }
            cudaError_t e = solve_batch(G, C, H, W, w_dtype == ISPA_BF16 ? ElemType::BF16 : ElemType::F32, DW, M, Y, P,
                                        reinterpret_cast<float *>(Yb + (size_t)z0 * mat),
                                        reinterpret_cast<float *>(Pb + (size_t)z0 * mat), split + 6 * (size_t)z0 * nD,
                                        terms + 5 * (size_t)z0 * eps_parts(D), eps_parts(D), layer_status + l0 + z0,
                                        eps + l0 + z0, err_terms ? err_terms + 2 * (size_t)(l0 + z0) : nullptr,
                                        w_new ? &WN : nullptr, D, lambda, bs, flag, ss);
            if (e != cudaSuccess) return cuda_fail(e, "absorb solve");
        }
        if (nsub > 1) {
            for (int i = 0; i < nsub - 1; ++i) {
                CUDA_CHECK_RET(cudaEventRecord(side->join[i], side->st[i]), "cudaEventRecord (join)");
                CUDA_CHECK_RET(cudaStreamWaitEvent(s, side->join[i], 0), "cudaStreamWaitEvent (join)");
            }
        }
    }
    return ISPA_OK;
}

int ispa_absorb_error(const ispa_stats *per_layer, int n_layers, const void *const *w_o, ispa_dtype w_dtype,
                      const float *const *dW, float *eps, double *err_terms, void *ws, size_t ws_bytes,
                      ispa_stream_t stream) {
    g_last_error.clear();
    if (n_layers < 0) return fail(ISPA_ERR_INVALID_ARG, "n_layers < 0");
    if (n_layers == 0) return ISPA_OK;
    if (!per_layer || !w_o || !dW || !eps) return fail(ISPA_ERR_INVALID_ARG, "per_layer, w_o, dW and eps are required");
    if (w_dtype != ISPA_BF16 && w_dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad w_dtype");
    const int D = per_layer[0].D;
    if (D <= 0 || D % 64 != 0) return fail(ISPA_ERR_UNSUPPORTED, "D=%d: needs D %% 64 == 0", D);
    for (int l = 0; l < n_layers; ++l) {
        int rc = check_stats(&per_layer[l], D);
        if (rc != ISPA_OK) return fail(rc, "layer %d: %s", l, g_last_error.c_str());
        if (!w_o[l]) return fail(ISPA_ERR_INVALID_ARG, "w_o[%d] is NULL", l);
        if (!dW[l]) return fail(ISPA_ERR_INVALID_ARG, "dW[%d] is NULL", l);
        if (!aligned(dW[l], 16)) return fail(ISPA_ERR_INVALID_ARG, "dW[%d] must be 16-byte aligned", l);
    }
    int rc = check_ws(ws, ws_bytes, solve_ws_bytes(n_layers, D));
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // workspace layout as for the solve (the M block is unused here)
    const size_t mat = (size_t)D * D * sizeof(float);
    const int bmax = std::min(n_layers, kMaxBatch);
    char *wsb = static_cast<char *>(ws);
    char *Yb = wsb + (size_t)bmax * mat, *Pb = wsb + 2 * (size_t)bmax * mat;
    float *split = reinterpret_cast<float *>(wsb + 3 * (size_t)bmax * mat);
    double *terms = reinterpret_cast<double *>(wsb + 9 * (size_t)bmax * mat);
    int *flag = nullptr;
    rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    for (int l0 = 0; l0 < n_layers; l0 += kMaxBatch) {
        const int b = std::min(kMaxBatch, n_layers - l0);
        PtrBatch G, C, H, W, DW, Y, P;
        for (int z = 0; z < b; ++z) {
            const ispa_stats &st = per_layer[l0 + z];
            G.p[z] = st.G; C.p[z] = st.C; H.p[z] = st.H;
            W.p[z] = const_cast<void *>(w_o[l0 + z]);
            DW.p[z] = const_cast<float *>(dW[l0 + z]);
            Y.p[z] = Yb + (size_t)z * mat;
            P.p[z] = Pb + (size_t)z * mat;
        }
        cudaError_t e = error_batch(G, C, H, W, w_dtype == ISPA_BF16 ? ElemType::BF16 : ElemType::F32, DW, Y, P,
                                    reinterpret_cast<float *>(Yb), reinterpret_cast<float *>(Pb), split, terms,
                                    eps_parts(D), eps + l0, err_terms ? err_terms + 2 * (size_t)l0 : nullptr, D, b, flag,
                                    s);
        if (e != cudaSuccess) return cuda_fail(e, "absorb error");
    }
    return ISPA_OK;
}

int ispa_quantize_w8(const void *w, ispa_dtype w_dtype, int d_in, int d_out, signed char *wq_t, float *w_scale,
                     ispa_stream_t stream) {
    g_last_error.clear();
    if (!w || !wq_t || !w_scale) return fail(ISPA_ERR_INVALID_ARG, "w, wq_t and w_scale are required");
    if (w_dtype != ISPA_BF16 && w_dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad w_dtype");
    if (d_in <= 0 || d_out <= 0 || d_in % 128 || d_out % 128)
        return fail(ISPA_ERR_UNSUPPORTED, "d_in=%d d_out=%d: both must be positive multiples of 128", d_in, d_out);
    if (!aligned(wq_t, 16)) return fail(ISPA_ERR_INVALID_ARG, "wq_t must be 16-byte aligned");
    cudaError_t e = launch_quant_cols(w, w_dtype == ISPA_BF16 ? ElemType::BF16 : ElemType::F32, d_in, d_out,
                                      reinterpret_cast<int8_t *>(wq_t), w_scale,
                                      reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "weight quantisation");
    return ISPA_OK;
}

int ispa_project_w8a8(const void *a, int n, int d_in, const signed char *wq_t, const float *w_scale, int d_out,
                      void *y, void *ws, size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    if (n < 0) return fail(ISPA_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return ISPA_OK;
    if (!a || !wq_t || !w_scale || !y) return fail(ISPA_ERR_INVALID_ARG, "a, wq_t, w_scale and y are required");
    if (d_in <= 0 || d_out <= 0 || d_in % 128 || d_out % 128)
        return fail(ISPA_ERR_UNSUPPORTED, "d_in=%d d_out=%d: both must be positive multiples of 128", d_in, d_out);
    if (!aligned(a, 16) || !aligned(y, 16) || !aligned(wq_t, 16))
        return fail(ISPA_ERR_INVALID_ARG, "a, y and wq_t must be 16-byte aligned");
    int rc = check_ws(ws, ws_bytes, w8a8_ws_bytes(n, d_in));
    if (rc != ISPA_OK) return rc;
    int *flag = nullptr;
    rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    int8_t *q_a = static_cast<int8_t *>(ws);
    float *s_a = reinterpret_cast<float *>(static_cast<char *>(ws) + align_up((size_t)n * d_in, 256));
    cudaError_t e = launch_project_w8a8(a, n, d_in, reinterpret_cast<const int8_t *>(wq_t), w_scale, d_out, y, q_a,
                                        s_a, flag, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "W8A8 projection");
    return ISPA_OK;
}

int ispa_select_layers(const float *eps_host, int n_layers, int K, int *idx_out, unsigned char *is_local) {
    g_last_error.clear();
    if (n_layers < 0) return fail(ISPA_ERR_INVALID_ARG, "n_layers < 0");
    if (K < 0) return fail(ISPA_ERR_INVALID_ARG, "K < 0");
    if (n_layers > 0 && !eps_host) return fail(ISPA_ERR_INVALID_ARG, "eps_host is NULL");
    std::vector<int> order(n_layers);
    for (int l = 0; l < n_layers; ++l) order[l] = l;
    auto key = [&](int l) {
        const float e = eps_host[l];
        return e != e ? INFINITY : e;   // NaN ranks last
    };
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        const float ka = key(a), kb = key(b);
        if (ka < kb) return true;
        if (kb < ka) return false;
        return a < b;
    });
    const int k = std::min(K, n_layers);
    if (idx_out)
        for (int i = 0; i < k; ++i) idx_out[i] = order[i];
    if (is_local) {
        for (int l = 0; l < n_layers; ++l) is_local[l] = 0;
        for (int i = 0; i < k; ++i) is_local[order[i]] = 1;
    }
    return ISPA_OK;
}

int ispa_rewarm_check(const float *live_history, int n_chunks, int n_layers, double ratio, double min_rise,
                      unsigned char *fired) {
    g_last_error.clear();
    if (n_chunks < 0 || n_layers < 0) return fail(ISPA_ERR_INVALID_ARG, "n_chunks and n_layers must be >= 0");
    if (n_layers > 0 && !fired) return fail(ISPA_ERR_INVALID_ARG, "fired is NULL");
    if (n_chunks > 0 && n_layers > 0 && !live_history) return fail(ISPA_ERR_INVALID_ARG, "live_history is NULL");
    if (!(ratio >= 0.0) || !(min_rise >= 0.0)) return fail(ISPA_ERR_INVALID_ARG, "ratio and min_rise must be >= 0");
    int count = 0;
    for (int l = 0; l < n_layers; ++l) {
        fired[l] = 0;
        if (n_chunks < 2) continue;
        const float latest = live_history[(size_t)(n_chunks - 1) * n_layers + l];
        if (latest != latest) continue;   // not monitored in the latest chunk
        double lowest = INFINITY;
        bool seen = false;
        for (int c = 0; c < n_chunks - 1; ++c) {
            const float e = live_history[(size_t)c * n_layers + l];
            if (e != e) continue;
            seen = true;
            lowest = std::min(lowest, (double)e);
        }
        if (seen && (double)latest > ratio * lowest && (double)latest > lowest + min_rise) {
            fired[l] = 1;
            ++count;
        }
    }
    return count;
}

int ispa_local_attn(const ispa_attn_desc *desc, const void *q, const void *k_loc, const void *v_loc, void *o,
                    float *lse, const void *w_new, void *y, void *ws, size_t ws_bytes, ispa_stream_t stream) {
    g_last_error.clear();
    int rc = check_desc(desc, false);
    if (rc != ISPA_OK) return rc;
    if (desc->n_q > 0 && (!q || !o)) return fail(ISPA_ERR_INVALID_ARG, "q and o are required");
    if (desc->n_kv > 0 && (!k_loc || !v_loc)) return fail(ISPA_ERR_INVALID_ARG, "k_loc and v_loc are required");
    if ((w_new == nullptr) != (y == nullptr)) return fail(ISPA_ERR_INVALID_ARG, "w_new and y go together");
    for (const void *p : {q, k_loc, v_loc, (const void *)o, w_new, (const void *)y})
        if (p && !aligned(p, 16)) return fail(ISPA_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = desc->heads * desc->head_dim;
    // lse is optional for the caller but the kernels always write one: park it in ws.
    float *lse_out = lse;
    size_t need = 0;
    if (!lse) need += align_up((size_t)desc->heads * desc->n_q * sizeof(float), 256);
    rc = check_ws(ws, ws_bytes, need);
    if (rc != ISPA_OK) return rc;
    if (!lse) lse_out = static_cast<float *>(ws);
    if (desc->n_q == 0) return ISPA_OK;
    rc = run_attention(desc, q, k_loc, v_loc, o, lse_out, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, true, s);
    if (rc != ISPA_OK) return rc;
    if (w_new) {
        if (desc->dtype == ISPA_BF16 && D % 128 == 0) {
            int *flag = nullptr;
            rc = device_error_flag(&flag);
            if (rc != ISPA_OK) return rc;
            CUDA_CHECK_RET(launch_gemm_bf16(o, w_new, y, desc->n_q, D, D, flag, s), "projection GEMM (tcgen05)");
        } else {
            const ElemType t = desc->dtype == ISPA_BF16 ? ElemType::BF16 : ElemType::F32;
            GemmDesc g{desc->n_q, D, D, D, D, D, true, false, t, t, t, 1.f, 0.f, false, 1};
            GemmBatch b;
            b.A[0] = o; b.B[0] = w_new; b.C[0] = y;
            CUDA_CHECK_RET(launch_gemm_simt(g, b, s), "projection GEMM");
        }
    }
    return ISPA_OK;
}

int ispa_project(const void *a, int n, int d_in, const void *w, int d_out, void *y, ispa_dtype dtype,
                 ispa_stream_t stream) {
    g_last_error.clear();
    if (n < 0 || d_in <= 0 || d_out <= 0) return fail(ISPA_ERR_INVALID_ARG, "bad sizes n=%d d_in=%d d_out=%d", n, d_in, d_out);
    if (dtype != ISPA_BF16 && dtype != ISPA_FP32) return fail(ISPA_ERR_INVALID_ARG, "bad dtype");
    if (n == 0) return ISPA_OK;
    if (!a || !w || !y) return fail(ISPA_ERR_INVALID_ARG, "a, w and y are required");
    if (!aligned(a, 16) || !aligned(w, 16) || !aligned(y, 16)) return fail(ISPA_ERR_INVALID_ARG, "a, w and y must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == ISPA_BF16 && d_in % 128 == 0 && d_out % 128 == 0) {
        int *flag = nullptr;
        int rc = device_error_flag(&flag);
        if (rc != ISPA_OK) return rc;
        CUDA_CHECK_RET(launch_gemm_bf16(a, w, y, n, d_out, d_in, flag, s), "projection GEMM (tcgen05)");
    } else {
        const ElemType t = dtype == ISPA_BF16 ? ElemType::BF16 : ElemType::F32;
        GemmDesc g{n, d_out, d_in, d_in, d_out, d_out, true, false, t, t, t, 1.f, 0.f, false, 1};
        GemmBatch b;
        b.A[0] = a; b.B[0] = w; b.C[0] = y;
        CUDA_CHECK_RET(launch_gemm_simt(g, b, s), "projection GEMM");
    }
    return ISPA_OK;
}

int ispa_set_attn_kernel(int choice) {
    if (choice != ISPA_ATTN_AUTO && choice != ISPA_ATTN_SINGLE && choice != ISPA_ATTN_PAIR &&
        choice != ISPA_ATTN_TWO_GROUP)
        return fail(ISPA_ERR_INVALID_ARG, "ispa_set_attn_kernel: unknown choice %d", choice);
    return g_attn_kernel.exchange(choice);
}

int ispa_device_status(ispa_stream_t stream) {
    g_last_error.clear();
    int *flag = nullptr;
    int rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    CUDA_CHECK_RET(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    int v = 0;
    CUDA_CHECK_RET(cudaMemcpy(&v, flag, sizeof(int), cudaMemcpyDeviceToHost), "read device flag");
    if (v != 0) {
        const int zero = 0;
        CUDA_CHECK_RET(cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice), "clear device flag");
        return fail(v, "a kernel reported device error %d", v);
    }
    return ISPA_OK;
}

int ispa_selftest_bounded_wait(unsigned limit_us, ispa_stream_t stream) {
    g_last_error.clear();
    if (limit_us < 1 || limit_us > 1000000) return fail(ISPA_ERR_INVALID_ARG, "limit_us must be in [1, 1e6]");
    int *flag = nullptr;
    int rc = device_error_flag(&flag);
    if (rc != ISPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    bounded_wait_selftest_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull, flag); note_launch();
    CUDA_CHECK_RET(cudaGetLastError(), "selftest launch");
    return ISPA_OK;
}

}  // extern "C"
