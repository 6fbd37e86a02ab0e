// y = A W on the sm_100a tensor cores, bf16 operands, float32 accumulation, bf16 output: the
// output projection of an L-layer with its updated weights, y = A_loc W_new [ISPA §3.1 step 3,
// §3.3].
//
// A [M][K] row-major (the attention output, K-major operand), W [K][N] row-major (the
// projection stored [D_in, D_out], MN-major operand), y [M][N] row-major. Persistent CTAs (one
// per SM) walk the 128x128 output tiles, K in steps of 64 through a 4-stage TMA ring (128-byte
// swizzle, no multicast); warp 0 TMA, warp 1 MMA into two TMEM accumulators in turn, warps 4..7
// epilogue. Rows of A beyond M are zero-filled by TMA and their outputs are not stored.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;
constexpr int kKStep = 64;
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kABytes = kTile * kKStep * 2;      // 16 KB
constexpr int kBBytes = kKStep * kTile * 2;      // 16 KB: two 64x64 boxes
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmem = kBarOff + 128;

struct ProjParams {
    bf16 *y;
    int M, N, K;
    int *err_flag;
};

// Persistent: one CTA per SM takes tiles t = blockIdx.x, + gridDim.x, ... (row tiles outermost).
// Warp 0 streams the k-steps through the stage ring (running ahead into the next tile), warp 1
// issues the MMAs into one of two TMEM accumulators, warps 4..7 drain the other, so a tile's
// epilogue (conversion to bf16, stores) overlaps the next tile's MMAs.
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB, const ProjParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (ptx::smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(p.err_flag, 0, ISPA_ERR_UNSUPPORTED);
        return;
    }
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *acc_full = empty + kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *done_bar = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int gx = p.N / kTile, gy = (p.M + kTile - 1) / kTile;
    const int ntiles = gx * gy;
    const int n_k = (p.K + kKStep - 1) / kKStep;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], 4);
        }
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 2 * kTile);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // producer and MMA warps stay converged; one elected lane issues (uniform registers)
    if (warp == 0) {
        const uint64_t pol_a = ptx::policy_evict_normal();
        const uint64_t pol_b = ptx::policy_evict_last();
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int m0 = (t / gx) * kTile, n0 = (t % gx) * kTile;
            for (int kt = 0; kt < n_k; ++kt, ++it) {
                const int s = it % kStages;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&empty[s], ((it / kStages) & 1) ^ 1,
                                                                     kWaitLimitNs, p.err_flag, abort_flag));
                if (!ok) break;
                uint8_t *base = smem + s * kStageBytes;
                ptx::mbar_arrive_expect_tx_warp(&full[s], kStageBytes);
                const int k0 = kt * kKStep;
                ptx::tma_load_2d_warp(base, &tA, &full[s], k0, m0, pol_a);
#pragma unroll
                for (int b = 0; b < 2; ++b)
                    ptx::tma_load_2d_warp(base + kABytes + b * (kKStep * 128), &tB, &full[s], n0 + b * 64, k0, pol_b);
            }
        }
        if (!ok) {
            // let copies in flight land before the CTA can exit (bounded)
            const uint64_t t0 = ptx::globaltimer_ns();
            while (ptx::globaltimer_ns() - t0 < 2000000ull) {
            }
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc = ptx::make_idesc_bf16(kTile, kTile, false, true);
        const uint32_t sbase = ptx::smem_u32(smem);
        int it = 0, i = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++i) {
            const int b = i & 1;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&acc_empty[b], ((i >> 1) & 1) ^ 1, kWaitLimitNs,
                                                                 p.err_flag, abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + (uint32_t)b * kTile;
            for (int kt = 0; kt < n_k; ++kt, ++it) {
                const int s = it % kStages;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&full[s], (it / kStages) & 1, kWaitLimitNs,
                                                                     p.err_flag, abort_flag));
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t a = sbase + s * kStageBytes, bb = a + kABytes;
#pragma unroll
                for (int kk = 0; kk < kKStep / 16; ++kk) {
                    const uint64_t da = ptx::make_sdesc_sw128(a + kk * 32, 16, 1024);
                    const uint64_t db = ptx::make_sdesc_sw128(bb + kk * 2048, kKStep * 128, 1024);
                    ptx::umma_f16_ss_warp(d, da, db, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::umma_commit_warp(&empty[s]);
            }
            if (!ok) break;
            ptx::umma_commit_warp(&acc_full[b]);
        }
        if (!ok) {
            if (lane == 0) *abort_flag = 1;
            __threadfence_block();
        }
        // every MMA issued has completed before tensor memory is released
        ptx::umma_commit_warp(done_bar);
        ptx::mbar_wait_bounded(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
    } else if (warp >= 4) {
        const int wq = warp - 4;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        int i = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
            const int m0 = (t / gx) * kTile, n0 = (t % gx) * kTile;
            const int b = i & 1;
            const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&acc_full[b], (i >> 1) & 1, kWaitLimitNs,
                                                                           p.err_flag, abort_flag)) &&
                            !*abort_flag;
            if (!ok) break;
            ptx::tc_fence_after();
            const int gm = m0 + r;
            bf16 *yrow = p.y + (size_t)gm * p.N + n0;
            const uint32_t tbuf = tmem + (uint32_t)b * kTile + lane_off;
#pragma unroll 1
            for (int c = 0; c < kTile / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tbuf + c * 32, v);
                ptx::tmem_wait_ld();
                if (c == kTile / 32 - 1) {
                    // the accumulator is in registers: hand it back to the MMA warp
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[b]);
                }
                if (gm < p.M) {
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1]));
                        pk[q] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(yrow + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 2 * kTile);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [rows][cols] bf16 row-major, box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int rows, int cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// y[M][N] = A[M][K] W[K][N], bf16 row-major in and out. N and K multiples of 128 and 64.
cudaError_t launch_gemm_bf16(const void *A, const void *W, void *y, int M, int N, int K, int *err_flag,
                             cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    if (N % kTile || K % kKStep) return cudaErrorInvalidValue;
    CUtensorMap ta, tb;
    if (!make_map(&ta, A, M, K, kTile) || !make_map(&tb, W, K, N, kKStep)) return cudaErrorInvalidValue;
    ProjParams p;
    p.y = static_cast<bf16 *>(y);
    p.M = M; p.N = N; p.K = K;
    p.err_flag = err_flag;
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int tiles = (N / kTile) * ((M + kTile - 1) / kTile);
    gemm_bf16_kernel<<<tiles < sms ? tiles : sms, kThreads, kSmem, s>>>(ta, tb, p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace ispa
