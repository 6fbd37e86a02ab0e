// Warmup call (split attention + fused ridge statistics) for callers that cannot allocate.
//
// ispa_attn_split needs a workspace for the bf16 operands A_loc and R that the attention
// epilogue hands to the statistics GEMM. Some callers cannot provide one: they run where
// cudaMalloc (or any allocator) is not available to them, e.g. inside a host framework that
// owns all device memory and only passes in the step's inputs and outputs, or in a plugin
// whose interface has no workspace argument. ispa_attn_split_noalloc keeps that handoff in
// a file-scope device array instead, so the call allocates nothing and needs no workspace.
//
// The array is 2 x 16 MiB (one slot per operand) and is held by every GPU that loads the
// library, until the process exits. Every call shares it: calls whose kernels overlap on
// the GPU (different streams, or different host threads on one device) race on it and must
// be serialised by the caller. Nothing in it needs to start at zero: each call writes every
// operand element it later reads.
#include <mutex>

#include "common.cuh"

namespace ispa {
int record_error(int code, const char *msg);   // api.cu: sets ispa_last_error()
}

namespace {

constexpr size_t kOperandSlotBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[2 * kOperandSlotBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device. Host code must not pass the
// symbol itself to a kernel: on the host it names a stand-in, not device memory.
int scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ispa::record_error(ISPA_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return ispa::record_error(ISPA_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return ispa::record_error(ISPA_ERR_CUDA, cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return ISPA_OK;
}

}  // namespace

extern "C" int ispa_attn_split_noalloc(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                                       void *o_full, float *lse_full, void *o_loc, float *lse_loc, void *o_hist,
                                       float *lse_hist, const ispa_stats *stats, ispa_stream_t stream) {
    if (!desc) return ispa::record_error(ISPA_ERR_INVALID_ARG, "desc is NULL");
    if (!stats) return ispa::record_error(ISPA_ERR_INVALID_ARG, "stats is NULL (without statistics no scratch is "
                                                                 "needed: call ispa_attn_split with ws = NULL)");
    if (desc->n_q < 0 || desc->heads <= 0 || desc->head_dim <= 0)
        return ispa::record_error(ISPA_ERR_INVALID_ARG, "bad sizes");
    const size_t esize = desc->dtype == ISPA_FP32 ? 4 : 2;
    const size_t operand = ispa::align_up((size_t)desc->n_q * desc->heads * desc->head_dim * esize, 256);
    if (operand > kOperandSlotBytes)
        return ispa::record_error(ISPA_ERR_UNSUPPORTED,
                                  "n_q * heads * head_dim too large for the static scratch: each statistics operand "
                                  "may use at most 16 MiB (8,388,608 bf16 or 4,194,304 float32 elements)");
    void *scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != ISPA_OK) return rc;
    return ispa_attn_split(desc, q, k, v, o_full, lse_full, o_loc, lse_loc, o_hist, lse_hist, stats, scratch,
                           2 * kOperandSlotBytes, stream);
}
