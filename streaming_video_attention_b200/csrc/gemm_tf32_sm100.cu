// Float32-accurate batched GEMM on the sm_100a tensor cores (3xTF32), for every product of the
// absorb solve [ISPA §3.2, §3.3]: Y = C W; the blocked factorisation's panels, trailing updates
// and rows of L^-1; the two products with L^-1; the Gram products W W^T and dW dW^T whose dots
// with G and H give the error traces.
//
// Each float32 operand X is split once into X_hi = X rounded to TF32 (11 significant bits)
// and X_lo = X - X_hi (exact in float32; the tensor core keeps its leading 11 bits). The
// product is accumulated in float32 TMEM as A_hi B_hi + A_hi B_lo + A_lo B_hi; the dropped
// A_lo B_lo term and the truncation of the lo parts are ~2^-22 relative, i.e. float32-level
// accuracy. A bf16 operand is exact in TF32 (lo = 0) and drops its lo terms (two bf16 operands:
// one term).
//
// Layouts: both MMA operands are K-major (32-bit K-major tiles with the 128-byte swizzle):
// A split as [batch][M][K], B split *and transposed* as [batch][N][K] (the split kernel for B
// writes B^T), so C = A B = A (B^T)^T. C float32 row-major with given row and batch strides,
// overwritten or subtracted from. The split operands are contiguous batches in the workspace,
// so one 3-D tensor map covers all layers. Persistent CTAs (one per SM) walk 128 x 256 output
// tiles (128 x 128 where N or the tile count calls for it); K in steps of 32 through a 2- or
// 3-stage ring; warp 0 TMA, warp 1 MMA (kind::tf32, K = 8 per instruction) into two TMEM
// accumulators in turn, warps 4..7 epilogue.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;
constexpr int kKStep = 32;                      // fp32 elements per stage = one 128-byte row
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kOpBytes = kTile * kKStep * 4;    // 16 KB: one A part (128 rows) per stage

__host__ __device__ constexpr uint32_t make_idesc_tf32(int M, int N, bool b_mn) {
    return (1u << 4)                    // D: f32
           | (2u << 7)                  // A: tf32
           | (2u << 10)                 // B: tf32
           | ((b_mn ? 1u : 0u) << 16)   // B major
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct Tf32Params {
    float *C;
    int M, N, K, batch;
    int a_lo;           // A_lo present (absent: A is exact in TF32, e.g. bf16)
    int b_lo;           // B_lo present
    int a_tri;          // 0: A full; 1: A lower triangular (k < m0 + 128); 2: A upper triangular (k >= m0)
    int sym;            // C = A A^T: only tiles with n0 <= m0 run (B is A)
    // optional trace partials: dot_out[z][tile] = sum over the tile of C_ij * X_z[i][j] (double),
    // X_z [M][N] row-major float32 or bf16 (one pointer per batch entry); with sym, an off-diagonal
    // tile also adds C_ij * X_z[j][i] (its mirror's share), and the skipped tiles write 0. A second
    // float32 X (dot_x2 -> dot_out2) may ride along. C is written only if write_c.
    PtrBatch dot_x, dot_x2;
    int has_dot, has_dot2;
    int dot_x_bf16;
    double *dot_out, *dot_out2;
    int write_c;
    // optional: C split for a later 3xTF32 product, hi = C rounded to TF32 and lo = C - hi,
    // [batch][M][N] (split_t = 0) or transposed [batch][N][M] (split_t = 1)
    float *split_hi, *split_lo;
    int split_t;
    size_t split_bstride;   // batch stride of the split (elements)
    // C row z, i, column j at C[z * c_bstride + i * ldc + j]; c_sub: C = C - A B
    size_t ldc, c_bstride;
    int c_sub;
    int *err_flag;
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u); }

// Stage layout for an output tile of 128 rows and BN columns (128 or 256): per k-step of 32, A_hi
// and A_lo (16 KB each), then B_hi and B_lo (BN x 128 bytes each). A 256-wide tile reads each A
// slice once for twice the columns: per SM and MMA cycle 96 instead of 128 bytes of operand reads.
template <int BN>
struct Tf32Cfg {
    static constexpr int kBBytes = BN * kKStep * 4;
    static constexpr int kStageBytes = 2 * kOpBytes + 2 * kBBytes;
    static constexpr int kStages = BN == 128 ? 3 : 2;
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmem = kBarOff + 256;   // barriers, TMEM slot, abort flag; 16 doubles at +128
};
static_assert(Tf32Cfg<128>::kSmem <= 232448 && Tf32Cfg<256>::kSmem <= 232448, "shared memory budget");

// Output tiles in the order the CTAs take them (t = blockIdx.x, + gridDim.x, ...): batch entries
// outermost, so that the tiles in flight at once share one layer's operands in L2; within a
// layer tile rows with the longest K range first when A is triangular, then columns.
struct TileId {
    int z, m, n;
    bool skip;   // wholly above the diagonal of a symmetric product
};
template <int BN>
__device__ __forceinline__ TileId tile_of(int t, int gx, int gy, int a_tri, int sym) {
    const int per_layer = gx * gy;
    TileId id;
    id.z = t / per_layer;
    const int rem = t - id.z * per_layer;
    const int mr = rem / gx;
    id.n = rem - mr * gx;
    id.m = a_tri == 1 ? gy - 1 - mr : mr;
    id.skip = sym && id.n * (BN / kTile) > id.m;
    return id;
}

// Persistent: one CTA per SM walks its share of the output tiles. Warp 0 streams the operand
// k-steps through the stage ring (running ahead into the next tile), warp 1 issues the MMAs
// into one of two TMEM accumulators, warps 4..7 drain the other: the epilogue of a tile (its
// dots, splits and stores) overlaps the MMAs of the next. Trace partials are kept per 128 x 128
// sub-tile whatever BN is.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tAh, const __grid_constant__ CUtensorMap tAl,
                   const __grid_constant__ CUtensorMap tBh, const __grid_constant__ CUtensorMap tBl,
                   const Tf32Params p) {
    using Cfg = Tf32Cfg<BN>;
    constexpr int kSub = BN / kTile;   // 128-column sub-tiles per tile
    extern __shared__ __align__(1024) uint8_t smem[];
    if (ptx::smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(p.err_flag, 0, ISPA_ERR_UNSUPPORTED);
        return;
    }
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *empty = full + Cfg::kStages;
    uint64_t *acc_full = empty + Cfg::kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *done_bar = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    double *red = reinterpret_cast<double *>(smem + Cfg::kBarOff + 128);   // [dot][sub][warp]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int gx = p.N / BN, gy = p.M / kTile, gx128 = p.N / kTile;
    const int ntiles = gx * gy * p.batch;
    const int n_kall = (p.K + kKStep - 1) / kKStep;
    const uint32_t stage_tx = (1 + p.a_lo) * kOpBytes + (1 + p.b_lo) * Cfg::kBBytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
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
        ptx::tmem_alloc(tmem_slot, 2 * BN);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // k-steps of a tile row: a triangular A is zero outside [kt0, kt1), and skipping exact zeros
    // changes no sum
    auto k_range = [&](int m0, int &kt0, int &n_k) {
        kt0 = p.a_tri == 2 ? m0 / kKStep : 0;
        const int kt1 = p.a_tri == 1 ? min(n_kall, (m0 + kTile) / kKStep) : n_kall;
        n_k = kt1 - kt0;
    };

    // producer and MMA warps stay converged; one elected lane issues (uniform registers)
    if (warp == 0) {
        const uint64_t pol = ptx::policy_evict_normal();
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileId id = tile_of<BN>(t, gx, gy, p.a_tri, p.sym);
            if (id.skip) continue;
            const int m0 = id.m * kTile, n0 = id.n * BN;
            int kt0, n_k;
            k_range(m0, kt0, n_k);
            for (int kt = 0; kt < n_k; ++kt, ++it) {
                const int s = it % Cfg::kStages;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&empty[s], ((it / Cfg::kStages) & 1) ^ 1,
                                                                     kWaitLimitNs, p.err_flag, abort_flag));
                if (!ok) break;
                uint8_t *base = smem + s * Cfg::kStageBytes;
                ptx::mbar_arrive_expect_tx_warp(&full[s], stage_tx);
                const int k0 = (kt0 + kt) * kKStep;
                ptx::tma_load_3d_warp(base, &tAh, &full[s], k0, m0, id.z, pol);
                if (p.a_lo) ptx::tma_load_3d_warp(base + kOpBytes, &tAl, &full[s], k0, m0, id.z, pol);
                ptx::tma_load_3d_warp(base + 2 * kOpBytes, &tBh, &full[s], k0, n0, id.z, pol);
                if (p.b_lo) ptx::tma_load_3d_warp(base + 2 * kOpBytes + Cfg::kBBytes, &tBl, &full[s], k0, n0, id.z, pol);
            }
        }
        if (!ok) {
            // let copies in flight land before the CTA can exit (bounded)
            const uint64_t t0 = ptx::globaltimer_ns();
            while (ptx::globaltimer_ns() - t0 < 2000000ull) {
            }
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc = make_idesc_tf32(kTile, BN, false);
        const uint32_t sbase = ptx::smem_u32(smem);
        int it = 0, i = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileId id = tile_of<BN>(t, gx, gy, p.a_tri, p.sym);
            if (id.skip) continue;
            int kt0, n_k;
            k_range(id.m * kTile, kt0, n_k);
            const int b = i & 1;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&acc_empty[b], ((i >> 1) & 1) ^ 1, kWaitLimitNs,
                                                                 p.err_flag, abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + (uint32_t)b * BN;
            for (int kt = 0; kt < n_k; ++kt, ++it) {
                const int s = it % Cfg::kStages;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&full[s], (it / Cfg::kStages) & 1, kWaitLimitNs,
                                                                     p.err_flag, abort_flag));
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t ah = sbase + s * Cfg::kStageBytes, al = ah + kOpBytes, bh = al + kOpBytes,
                               bl = bh + Cfg::kBBytes;
#pragma unroll
                for (int kk = 0; kk < kKStep / 8; ++kk) {
                    const uint64_t dah = ptx::make_sdesc_sw128(ah + kk * 32, 16, 1024);
                    const uint64_t dal = ptx::make_sdesc_sw128(al + kk * 32, 16, 1024);
                    const uint64_t dbh = ptx::make_sdesc_sw128(bh + kk * 32, 16, 1024);
                    uint32_t acc = (kt == 0 && kk == 0) ? 0u : 1u;
                    if (p.a_lo) {
                        ptx::umma_tf32_ss_warp(d, dal, dbh, idesc, acc);
                        acc = 1u;
                    }
                    if (p.b_lo) {
                        const uint64_t dbl = ptx::make_sdesc_sw128(bl + kk * 32, 16, 1024);
                        ptx::umma_tf32_ss_warp(d, dah, dbl, idesc, acc);
                        acc = 1u;
                    }
                    ptx::umma_tf32_ss_warp(d, dah, dbh, idesc, acc);
                }
                ptx::umma_commit_warp(&empty[s]);
            }
            if (!ok) break;
            ptx::umma_commit_warp(&acc_full[b]);
            ++i;
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
        const bool has_parts = p.has_dot || p.has_dot2;
        int i = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const TileId id = tile_of<BN>(t, gx, gy, p.a_tri, p.sym);
            const int z = id.z, m0 = id.m * kTile, n0 = id.n * BN;
            // partial of 128 x 128 sub-tile u of this tile
            const size_t part0 = ((size_t)z * gy + id.m) * gx128 + (size_t)id.n * kSub;
            if (id.skip) {
                // the mirror tiles account for these
                if (wq == 0 && lane == 0)
                    for (int u = 0; u < kSub; ++u) {
                        if (p.has_dot) p.dot_out[part0 + u] = 0.0;
                        if (p.has_dot2) p.dot_out2[part0 + u] = 0.0;
                    }
                continue;
            }
            const int b = i & 1;
            const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&acc_full[b], (i >> 1) & 1, kWaitLimitNs,
                                                                           p.err_flag, abort_flag)) &&
                            !*abort_flag;
            if (!ok) break;
            ptx::tc_fence_after();
            double part[kSub], part2[kSub];
#pragma unroll
            for (int u = 0; u < kSub; ++u) part[u] = part2[u] = 0.0;
            const int gm = m0 + r;
            float *crow = p.C + (size_t)z * p.c_bstride + (size_t)gm * p.ldc + n0;
            const size_t xrow = (size_t)gm * p.N + n0;
            const void *xz = p.has_dot ? p.dot_x.p[z] : nullptr;
            const float *x2z = p.has_dot2 ? static_cast<const float *>(p.dot_x2.p[z]) : nullptr;
            const uint32_t tbuf = tmem + (uint32_t)b * BN + lane_off;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tbuf + c * 32, v);
                ptx::tmem_wait_ld();
                if (c == BN / 32 - 1) {
                    // the accumulator is in registers: hand it back to the MMA warp
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[b]);
                }
                const int u = c / (kTile / 32);              // sub-tile of this chunk
                const int nt = id.n * kSub + u;              // its 128-column tile index
                // a symmetric product keeps only sub-tiles on or below the diagonal; an
                // off-diagonal one also takes its mirror's share of the dots
                if (p.sym && nt > id.m) continue;
                const bool mirror = p.sym && nt != id.m;
                double pa = 0.0, pb = 0.0;
                if (p.has_dot) {
                    // products of two floats are exact in double; summed in a fixed order. The row's
                    // 32 values are read as 16-byte vectors (N is a multiple of 128).
                    float x[32];
                    if (p.dot_x_bf16) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const bf16 *>(xz) + xrow + c * 32);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint4 q4 = src[w];
                            const uint32_t ww[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                x[8 * w + 2 * e] = __uint_as_float(ww[e] << 16);
                                x[8 * w + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
                            }
                        }
                    } else {
                        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(xz) + xrow + c * 32);
#pragma unroll
                        for (int w = 0; w < 8; ++w) {
                            const float4 q4 = src[w];
                            x[4 * w] = q4.x; x[4 * w + 1] = q4.y; x[4 * w + 2] = q4.z; x[4 * w + 3] = q4.w;
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 32; ++q) pa += (double)__uint_as_float(v[q]) * (double)x[q];
                    if (mirror) {
                        // X[n0 + c*32 + q][gm]: the warp's 32 rows read one 128-byte run per q
                        const float *xt = static_cast<const float *>(xz) + (size_t)(n0 + c * 32) * p.N + gm;
#pragma unroll
                        for (int q = 0; q < 32; ++q) x[q] = xt[(size_t)q * p.N];
#pragma unroll
                        for (int q = 0; q < 32; ++q) pa += (double)__uint_as_float(v[q]) * (double)x[q];
                    }
                }
                if (p.has_dot2) {
                    float x[32];
                    const float4 *src = reinterpret_cast<const float4 *>(x2z + xrow + c * 32);
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        const float4 q4 = src[w];
                        x[4 * w] = q4.x; x[4 * w + 1] = q4.y; x[4 * w + 2] = q4.z; x[4 * w + 3] = q4.w;
                    }
#pragma unroll
                    for (int q = 0; q < 32; ++q) pb += (double)__uint_as_float(v[q]) * (double)x[q];
                    if (mirror) {
                        const float *xt = x2z + (size_t)(n0 + c * 32) * p.N + gm;
#pragma unroll
                        for (int q = 0; q < 32; ++q) x[q] = xt[(size_t)q * p.N];
#pragma unroll
                        for (int q = 0; q < 32; ++q) pb += (double)__uint_as_float(v[q]) * (double)x[q];
                    }
                }
#pragma unroll
                for (int w = 0; w < kSub; ++w)
                    if (w == u) {
                        part[w] += pa;
                        part2[w] += pb;
                    }
                if (p.split_hi) {
                    if (p.split_t) {
                        // column n0 + c*32 + q of C is row n of the transposed split: the warp's
                        // 32 rows write one 128-byte run per q
                        const size_t base = (size_t)z * p.split_bstride + (size_t)(n0 + c * 32) * p.M + gm;
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const float x = __uint_as_float(v[q]), h = tf32_hi(x);
                            p.split_hi[base + (size_t)q * p.M] = h;
                            p.split_lo[base + (size_t)q * p.M] = x - h;
                        }
                    } else {
                        float *hrow = p.split_hi + (size_t)z * p.split_bstride + (size_t)gm * p.N + n0 + c * 32;
                        float *lrow = p.split_lo + (size_t)z * p.split_bstride + (size_t)gm * p.N + n0 + c * 32;
#pragma unroll
                        for (int q = 0; q < 32; q += 4) {
                            float h[4], l[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float x = __uint_as_float(v[q + e]);
                                h[e] = tf32_hi(x);
                                l[e] = x - h[e];
                            }
                            *reinterpret_cast<float4 *>(hrow + q) = make_float4(h[0], h[1], h[2], h[3]);
                            *reinterpret_cast<float4 *>(lrow + q) = make_float4(l[0], l[1], l[2], l[3]);
                        }
                    }
                }
                if (p.write_c) {
                    if (p.c_sub) {
                        float4 old[8];
#pragma unroll
                        for (int w = 0; w < 8; ++w) old[w] = *reinterpret_cast<const float4 *>(crow + c * 32 + 4 * w);
#pragma unroll
                        for (int w = 0; w < 8; ++w)
                            *reinterpret_cast<float4 *>(crow + c * 32 + 4 * w) =
                                make_float4(old[w].x - __uint_as_float(v[4 * w]), old[w].y - __uint_as_float(v[4 * w + 1]),
                                            old[w].z - __uint_as_float(v[4 * w + 2]),
                                            old[w].w - __uint_as_float(v[4 * w + 3]));
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; q += 4)
                            *reinterpret_cast<float4 *>(crow + c * 32 + q) =
                                make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]), __uint_as_float(v[q + 2]),
                                            __uint_as_float(v[q + 3]));
                    }
                }
            }
            if (has_parts) {
                // each sub-tile's partials: warp sums, then warp 4 adds the four warps' sums in order
                // (a sub-tile above the diagonal of a symmetric product sums to 0)
#pragma unroll
                for (int u = 0; u < kSub; ++u) {
                    for (int o = 16; o > 0; o >>= 1) {
                        part[u] += __shfl_down_sync(0xffffffffu, part[u], o);
                        part2[u] += __shfl_down_sync(0xffffffffu, part2[u], o);
                    }
                    if (lane == 0) {
                        red[(0 * kSub + u) * 4 + wq] = part[u];
                        red[(1 * kSub + u) * 4 + wq] = part2[u];
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (wq == 0 && lane == 0)
                    for (int u = 0; u < kSub; ++u) {
                        const double *r1 = red + (0 * kSub + u) * 4, *r2 = red + (1 * kSub + u) * 4;
                        if (p.has_dot) p.dot_out[part0 + u] = ((r1[0] + r1[1]) + r1[2]) + r1[3];
                        if (p.has_dot2) p.dot_out2[part0 + u] = ((r2[0] + r2[1]) + r2[2]) + r2[3];
                    }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            ++i;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 2 * BN);
    }
}

// X_hi = X rounded to TF32 (round to nearest, ties away from zero on the 13 dropped bits),
// X_lo = X - X_hi, for a batch of float32 or bf16 [rows][cols] matrices with row stride ld,
// written to [rows][cols] arrays dst_bstride elements apart. bf16 inputs are exact in TF32: lo
// is not written.
__device__ __forceinline__ float tf32_round(float x) { return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u); }

template <typename T>
__global__ void split_tf32_kernel(PtrBatch src, float *hi, float *lo, int rows, int cols, size_t ld,
                                  size_t dst_bstride) {
    const int z = blockIdx.y;
    const T *s = static_cast<const T *>(src.p[z]);
    float *h = hi + (size_t)z * dst_bstride;
    float *l = lo ? lo + (size_t)z * dst_bstride : nullptr;
    const size_t n = (size_t)rows * cols;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t si = ld == (size_t)cols ? i : (i / cols) * ld + i % cols;
        const float x = to_f32(s[si]);
        const float xh = tf32_round(x);
        h[i] = xh;
        if (l) l[i] = x - xh;
    }
}

// The same split of a batch of [rows][cols] matrices (row stride ld), written transposed
// ([cols][rows]) through a 32 x 32 shared-memory tile so that reads and writes stay coalesced.
template <typename T>
__global__ void split_tf32_transposed_kernel(PtrBatch src, float *hi, float *lo, int rows, int cols, size_t ld,
                                             size_t dst_bstride) {
    __shared__ float tile[32][33];
    const int z = blockIdx.z;
    const T *s = static_cast<const T *>(src.p[z]);
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        tile[i][threadIdx.x] = (r < rows && c < cols) ? to_f32(s[(size_t)r * ld + c]) : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < cols) {
            const float x = tile[threadIdx.x][i];
            const float xh = tf32_round(x);
            const size_t o = (size_t)z * dst_bstride + (size_t)c * rows + r;
            hi[o] = xh;
            if (lo) lo[o] = x - xh;
        }
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

// [batch][rows][cols] float32, box = (32 cols, box_rows rows, 1), 128-byte swizzle.
bool make_map(CUtensorMap *m, const float *ptr, int batch, int rows, int cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)rows * cols * 4};
    cuuint32_t box[3] = {32, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_split_tf32(const PtrBatch &src, ElemType t, float *hi, float *lo, int rows, int cols,
                              bool transpose, int batch, cudaStream_t s, size_t ld, size_t dst_bstride) {
    if (rows <= 0 || cols <= 0 || batch <= 0) return cudaSuccess;
    if (!ld) ld = cols;
    if (!dst_bstride) dst_bstride = (size_t)rows * cols;
    if (transpose) {
        const dim3 grid((cols + 31) / 32, (rows + 31) / 32, batch), block(32, 8);
        if (t == ElemType::BF16)
            split_tf32_transposed_kernel<bf16><<<grid, block, 0, s>>>(src, hi, nullptr, rows, cols, ld, dst_bstride);
        else split_tf32_transposed_kernel<float><<<grid, block, 0, s>>>(src, hi, lo, rows, cols, ld, dst_bstride);
    } else {
        const size_t n = (size_t)rows * cols;
        const int blocks = (int)std::min<size_t>((n + 255) / 256, 1024);
        if (t == ElemType::BF16)
            split_tf32_kernel<bf16><<<dim3(blocks, batch), 256, 0, s>>>(src, hi, nullptr, rows, cols, ld, dst_bstride);
        else split_tf32_kernel<float><<<dim3(blocks, batch), 256, 0, s>>>(src, hi, lo, rows, cols, ld, dst_bstride);
    }
    note_launch();
    return cudaGetLastError();
}

// C[z] = A[z] B[z] for z < batch; A given as (A_hi, A_lo or null) [batch][M][K], B as (B_hi,
// B_lo or null) transposed, [batch][N][K], all contiguous float32 (a null lo part: that operand
// is exact in TF32). M, N multiples of 128; K of 32. Options (Tf32Opts):
//   a_tri: 1 when A is lower triangular, 2 when upper triangular (then M = K): the zero part of
//          A is not read;
//   sym:   B is A (M = N): only the output tiles on and below the diagonal are formed;
//   dot_x / dot_out (and dot_x2 / dot_out2, float32): per batch entry z a [M][N] row-major X_z;
//          dot_out[z][t] = sum over output tile t (m-tile major) of C_ij * X_z[i][j] in double,
//          with sym also C_ij * X_z[j][i] off the diagonal (so the partials add up to
//          sum_ij (A A^T)_ij X_ij);
//   split_hi / split_lo: C's TF32 split for a later product, [batch][M][N] or with split_t
//          transposed [batch][N][M], split_bstride elements per batch entry (0: M*N);
//   ldc, c_bstride (0: N, M*N): C's row and batch strides (a block of a larger matrix);
//   c_sub: C = C - A B (the old C read in the epilogue);
//   write_c: C is written (always, when neither a dot nor a split is asked for).
cudaError_t launch_gemm_tf32x3(const float *Ah, const float *Al, const float *Bh, const float *Bl, float *C, int M,
                               int N, int K, int batch, int *err_flag, cudaStream_t s, const Tf32Opts &o) {
    if (M % kTile || N % kTile || K % kKStep || batch <= 0) return cudaErrorInvalidValue;
    if (o.sym && (M != N || o.dot_x_bf16 || o.a_tri)) return cudaErrorInvalidValue;
    // 256-wide tiles where N allows and they still give every SM two tiles or more (the A slices
    // are read once for twice the columns; the small products keep 128 for parallelism)
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int bn = (N % 256 == 0 && (long long)(M / kTile) * (N / 256) * batch >= 2LL * sms) ? 256 : 128;
    CUtensorMap ah, al, bh, bl;
    if (!make_map(&ah, Ah, batch, M, K, kTile) || !make_map(&al, Al ? Al : Ah, batch, M, K, kTile) ||
        !make_map(&bh, Bh, batch, N, K, bn) || !make_map(&bl, Bl ? Bl : Bh, batch, N, K, bn))
        return cudaErrorInvalidValue;
    Tf32Params p;
    p.C = C; p.M = M; p.N = N; p.K = K;
    p.a_lo = Al != nullptr;
    p.b_lo = Bl != nullptr;
    p.a_tri = (o.a_tri == 1 || o.a_tri == 2) && M == K ? o.a_tri : 0;
    p.sym = o.sym ? 1 : 0;
    p.has_dot = (o.dot_out && o.dot_x) ? 1 : 0;
    if (p.has_dot) p.dot_x = *o.dot_x;
    p.has_dot2 = (o.dot_out2 && o.dot_x2) ? 1 : 0;
    if (p.has_dot2) p.dot_x2 = *o.dot_x2;
    p.dot_x_bf16 = o.dot_x_bf16 ? 1 : 0;
    p.dot_out = o.dot_out;
    p.dot_out2 = o.dot_out2;
    p.split_hi = o.split_hi;
    p.split_lo = o.split_hi ? o.split_lo : nullptr;
    p.split_t = o.split_t ? 1 : 0;
    p.split_bstride = o.split_bstride ? o.split_bstride : (size_t)M * N;
    p.ldc = o.ldc ? o.ldc : (size_t)N;
    p.c_bstride = o.c_bstride ? o.c_bstride : (size_t)M * N;
    p.c_sub = o.c_sub ? 1 : 0;
    if (p.ldc % 4 || p.c_bstride % 4) return cudaErrorInvalidValue;
    if (p.split_hi && !p.split_lo) return cudaErrorInvalidValue;
    p.write_c = (o.write_c || !(p.has_dot || p.has_dot2 || p.split_hi)) ? 1 : 0;
    p.err_flag = err_flag;
    p.batch = batch;
    const long long tiles = (long long)(M / kTile) * (N / bn) * batch;
    const int grid = (int)(tiles < sms ? tiles : sms);
    if (bn == 256) {
        e = cudaFuncSetAttribute(gemm_tf32x3_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Tf32Cfg<256>::kSmem);
        if (e != cudaSuccess) return e;
        gemm_tf32x3_kernel<256><<<grid, kThreads, Tf32Cfg<256>::kSmem, s>>>(ah, al, bh, bl, p);
    } else {
        e = cudaFuncSetAttribute(gemm_tf32x3_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Tf32Cfg<128>::kSmem);
        if (e != cudaSuccess) return e;
        gemm_tf32x3_kernel<128><<<grid, kThreads, Tf32Cfg<128>::kSmem, s>>>(ah, al, bh, bl, p);
    }
    note_launch();
    return cudaGetLastError();
}

}  // namespace ispa
