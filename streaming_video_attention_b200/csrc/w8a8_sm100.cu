// W8A8 output projection of the L-layers: y = A W_new through int8 operands on the sm_100a
// tensor cores [ISPA §4.4: ISPA combined with 8-bit weights and activations for the linear
// layers; the quantisation scheme is not given].
//
// Scheme (a reading): symmetric int8, one float32 scale per activation row (token) and one per
// weight output column. scale = amax / 127; q = rint(x * (127 / amax)) clamped to [-127, 127]
// (round to nearest even, IEEE float32 division and multiplication); an all-zero slice has
// scale 0 and q = 0. The product accumulates exactly in int32 (tcgen05 kind::i8, |acc| <=
// 127 * 127 * K < 2^31 for K <= 133,000) and the epilogue forms
// y = bf16((float(acc) * s_row) * s_col). Every step is a plain float32 or integer operation,
// so the result is reproducible bit for bit.
//
// Kernels:
//   quant_rows_kernel  activations [n][K] (bf16) -> int8 [n][K] + scales [n]; one warp per row.
//   quant_cols_kernel  weights [K][N] (bf16 or float32) -> int8 [N][K] (transposed: K-major, the
//                      layout the MMA's B operand wants) + scales [N]; a CTA per 32 columns.
//   gemm_i8_kernel     y[M][N] from the two int8 operands, both K-major; persistent CTAs (one per
//                      SM) walk the 128x128 tiles, K in steps of 128 through a 4-stage TMA ring
//                      (128-byte swizzle, no multicast), a converged producer warp, a converged
//                      MMA warp issuing through elect.sync into two TMEM accumulators in turn,
//                      warps 4..7 epilogue (dequantise, bf16, store).
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;
constexpr int kKStep = 128;                      // int8 elements = bytes: one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kOpBytes = kTile * kKStep;         // 16 KB
constexpr int kStageBytes = 2 * kOpBytes;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmem = kBarOff + 128 + 1024;      // + slack for 1024-byte alignment

__device__ __forceinline__ float to_float(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_float(float x) { return x; }

__device__ __forceinline__ int quant1(float x, float inv) {
    const int q = __float2int_rn(__fmul_rn(x, inv));
    return max(-127, min(127, q));
}

// One warp per row of x [n][K] (K a multiple of 8, rows 16-byte aligned): amax, scale, int8 codes.
__global__ void quant_rows_kernel(const bf16 *__restrict__ x, int n, int K, int8_t *__restrict__ q,
                                  float *__restrict__ scale) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
    if (warp >= n) return;
    const uint4 *row = reinterpret_cast<const uint4 *>(x + (size_t)warp * K);   // 8 bf16 per vector
    const int nv = K / 8;
    float amax = 0.f;
    for (int v = lane; v < nv; v += 32) {
        const uint4 u = row[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
    uint2 *qrow = reinterpret_cast<uint2 *>(q + (size_t)warp * K);
    for (int v = lane; v < nv; v += 32) {
        const uint4 u = row[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int lo = quant1(__uint_as_float(w[i] << 16), inv);
            const int hi = quant1(__uint_as_float(w[i] & 0xFFFF0000u), inv);
            packed[i / 2] |= ((uint32_t)(lo & 0xFF) | ((uint32_t)(hi & 0xFF) << 8)) << (16 * (i % 2));
        }
        qrow[v] = make_uint2(packed[0], packed[1]);
    }
    if (lane == 0) scale[warp] = __fdiv_rn(amax, 127.f);
}

// K of the 8-bit split attention: one scale per (block, head), a block being up to 128 rows
// of one KV segment (segments in row order, each cut into blocks from its first row).
// k [n_kv][heads][128] bf16 -> k8 (same layout) + k_scale [heads][n_blocks]. One CTA per
// (block, head); thread t handles 8 columns (one 16-byte vector) of rows t/16, t/16 + 16, ...
__global__ void __launch_bounds__(256) quant_kblocks_kernel(const bf16 *__restrict__ k, int heads, SegmentList segs,
                                                            int n_blocks, int8_t *__restrict__ k8,
                                                            float *__restrict__ k_scale) {
    const int blk = blockIdx.x, head = blockIdx.y;
    int first = 0, r0 = 0, r1 = 0;
    for (int i = 0; i < segs.count; ++i) {
        const int nb = (segs.seg[i].end - segs.seg[i].begin + 127) / 128;
        if (blk < first + nb) {
            r0 = segs.seg[i].begin + (blk - first) * 128;
            r1 = min(r0 + 128, segs.seg[i].end);
            break;
        }
        first += nb;
    }
    const int v = threadIdx.x % 16, rb = threadIdx.x / 16;
    uint4 val[8];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + rb + 16 * i;
        val[i] = make_uint4(0u, 0u, 0u, 0u);
        if (r < r1) val[i] = *reinterpret_cast<const uint4 *>(k + ((size_t)r * heads + head) * 128 + v * 8);
        const uint32_t w[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
        }
    }
    __shared__ float red[8];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + rb + 16 * i;
        if (r >= r1) continue;
        const uint32_t w[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int lo = quant1(__uint_as_float(w[j] << 16), inv);
            const int hi = quant1(__uint_as_float(w[j] & 0xFFFF0000u), inv);
            packed[j / 2] |= ((uint32_t)(lo & 0xFF) | ((uint32_t)(hi & 0xFF) << 8)) << (16 * (j % 2));
        }
        *reinterpret_cast<uint2 *>(k8 + ((size_t)r * heads + head) * 128 + v * 8) = make_uint2(packed[0], packed[1]);
    }
    if (threadIdx.x == 0) k_scale[(size_t)head * n_blocks + blk] = __fdiv_rn(amax, 127.f);
}

// Weights w [K][N] row-major -> codes qt [N][K] and column scales [N]. CTA = 32 columns x 8
// row groups; pass 1 finds each column's amax, pass 2 quantises 32 x 128 tiles through shared
// memory so that both the reads of w and the writes of qt are coalesced.
template <typename T>
__global__ void quant_cols_kernel(const T *__restrict__ w, int K, int N, int8_t *__restrict__ qt,
                                  float *__restrict__ scale) {
    __shared__ float red[8][33];
    __shared__ float inv_s[32];
    __shared__ __align__(16) int8_t tile[32][128 + 16];   // rows of 144 bytes: 16-byte aligned chunks
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;   // 32 x 8 threads
    const int j0 = blockIdx.x * 32;
    const int j = j0 + tx;
    float amax = 0.f;
    for (int k = ty; k < K; k += 8) amax = fmaxf(amax, fabsf(to_float(w[(size_t)k * N + j])));
    red[ty][tx] = amax;
    __syncthreads();
    if (ty == 0) {
        float m = red[0][tx];
#pragma unroll
        for (int r = 1; r < 8; ++r) m = fmaxf(m, red[r][tx]);
        inv_s[tx] = m > 0.f ? __fdiv_rn(127.f, m) : 0.f;
        scale[j] = __fdiv_rn(m, 127.f);
    }
    __syncthreads();
    for (int k0 = 0; k0 < K; k0 += 128) {
        // load 128 rows x 32 columns, quantise, store transposed into the tile
        for (int kk = ty; kk < 128; kk += 8) tile[tx][kk] = (int8_t)quant1(to_float(w[(size_t)(k0 + kk) * N + j]), inv_s[tx]);
        __syncthreads();
        // write 32 rows of qt (columns j0..j0+31), 128 bytes each: 8 threads per row, 16 bytes each
        for (int r = threadIdx.x / 8; r < 32; r += 32) {
            const int part = threadIdx.x % 8;
            const uint4 v = *reinterpret_cast<const uint4 *>(&tile[r][part * 16]);
            *reinterpret_cast<uint4 *>(qt + (size_t)(j0 + r) * K + k0 + part * 16) = v;
        }
        __syncthreads();
    }
}

struct I8Params {
    bf16 *y;
    const float *row_scale;   // [M]
    const float *col_scale;   // [N]
    int M, N, K;
    int *err_flag;
};

// Instruction descriptor, kind::i8: D s32, A and B signed 8-bit, both K-major.
__host__ __device__ constexpr uint32_t make_idesc_s8(int M, int N) {
    return (2u << 4)                       // D format: s32
           | (1u << 7)                     // A format: signed 8-bit
           | (1u << 10)                    // B format: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_s8_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\t"
        "elect.sync r|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Persistent: one CTA per SM takes tiles t = blockIdx.x, + gridDim.x, ... (row tiles outermost);
// two TMEM accumulators in turn, so a tile's epilogue overlaps the next tile's MMAs.
__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB, const I8Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    const int n_k = p.K / kKStep;

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
                ptx::tma_load_2d_warp(base, &tA, &full[s], kt * kKStep, m0, pol_a);
                ptx::tma_load_2d_warp(base + kOpBytes, &tB, &full[s], kt * kKStep, n0, pol_b);
            }
        }
        if (!ok) {
            // let copies in flight land before the CTA can exit (bounded)
            const uint64_t t0 = ptx::globaltimer_ns();
            while (ptx::globaltimer_ns() - t0 < 2000000ull) {
            }
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc = make_idesc_s8(kTile, kTile);
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
                const uint32_t a = sbase + s * kStageBytes, bb = a + kOpBytes;
#pragma unroll
                for (int kk = 0; kk < kKStep / 32; ++kk) {   // 32 int8 = 32 bytes per MMA
                    const uint64_t da = ptx::make_sdesc_sw128(a + kk * 32, 16, 1024);
                    const uint64_t db = ptx::make_sdesc_sw128(bb + kk * 32, 16, 1024);
                    umma_s8_ss_warp(d, da, db, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
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
            const float sr = gm < p.M ? p.row_scale[gm] : 0.f;
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
                        const int cj = n0 + c * 32 + 2 * q;
                        const float y0 = __fmul_rn(__fmul_rn(__int2float_rn((int)v[2 * q]), sr), p.col_scale[cj]);
                        const float y1 = __fmul_rn(__fmul_rn(__int2float_rn((int)v[2 * q + 1]), sr), p.col_scale[cj + 1]);
                        __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
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

// [rows][K] int8 row-major, box = 128 bytes of K x 128 rows, 128-byte swizzle.
bool make_i8_map(CUtensorMap *m, const void *ptr, int rows, int K) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)kKStep, (cuuint32_t)kTile};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Weights [K][N] (bf16 or float32) -> int8 [N][K] + scales [N]. K, N multiples of 128 and 32.
cudaError_t launch_quant_cols(const void *w, ElemType t, int K, int N, int8_t *qt, float *scale, cudaStream_t s) {
    if (K % 128 || N % 32) return cudaErrorInvalidValue;
    if (t == ElemType::BF16)
        quant_cols_kernel<bf16><<<N / 32, 256, 0, s>>>(static_cast<const bf16 *>(w), K, N, qt, scale);
    else
        quant_cols_kernel<float><<<N / 32, 256, 0, s>>>(static_cast<const float *>(w), K, N, qt, scale);
    note_launch();
    return cudaGetLastError();
}

// y[M][N] = dequant(quant_rows(A)[M][K] x qt[N][K]^T): A bf16 [M][K]; q_a / s_a are scratch.
cudaError_t launch_project_w8a8(const void *A, int M, int K, const int8_t *qt, const float *col_scale, int N,
                                void *y, int8_t *q_a, float *s_a, int *err_flag, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    if (N % kTile || K % kKStep) return cudaErrorInvalidValue;
    quant_rows_kernel<<<(M + 7) / 8, 256, 0, s>>>(static_cast<const bf16 *>(A), M, K, q_a, s_a);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap ta, tb;
    if (!make_i8_map(&ta, q_a, M, K) || !make_i8_map(&tb, qt, N, K)) return cudaErrorInvalidValue;
    I8Params p;
    p.y = static_cast<bf16 *>(y);
    p.row_scale = s_a;
    p.col_scale = col_scale;
    p.M = M; p.N = N; p.K = K;
    p.err_flag = err_flag;
    e = cudaFuncSetAttribute(gemm_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int tiles = (N / kTile) * ((M + kTile - 1) / kTile);
    gemm_i8_kernel<<<tiles < sms ? tiles : sms, kThreads, kSmem, s>>>(ta, tb, p);
    note_launch();
    return cudaGetLastError();
}

// Q of the 8-bit split attention: q [n][heads][128] bf16 -> q8 (same layout) + q_scale
// [n][heads], one symmetric scale per (token, head): the row quantiser on n * heads rows.
cudaError_t launch_quant_q_i8(const void *q, int n, int heads, int8_t *q8, float *q_scale, cudaStream_t s) {
    const int rows = n * heads;
    if (rows <= 0) return cudaSuccess;
    quant_rows_kernel<<<(rows + 7) / 8, 256, 0, s>>>(static_cast<const bf16 *>(q), rows, 128, q8, q_scale);
    note_launch();
    return cudaGetLastError();
}

// K of the 8-bit split attention; segs in row order, n_blocks = their 128-row blocks.
cudaError_t launch_quant_k_i8(const void *k, int heads, const SegmentList &segs, int n_blocks, int8_t *k8,
                              float *k_scale, cudaStream_t s) {
    if (n_blocks <= 0) return cudaSuccess;
    quant_kblocks_kernel<<<dim3(n_blocks, heads), 256, 0, s>>>(static_cast<const bf16 *>(k), heads, segs, n_blocks, k8,
                                                                k_scale);
    note_launch();
    return cudaGetLastError();
}

}  // namespace ispa
