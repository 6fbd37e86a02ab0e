// Ridge statistics on the sm_100a tensor cores [ISPA §3.2; notes: Method]:
//   G += A^T A,  C += A^T R,  H += R^T R
// from the bf16 operands A = A_loc and R = A_full - A_loc, each [n, D] row-major (the
// layout the split-attention epilogue writes), accumulated in float32.
//
// D a multiple of 256 (every model shape here): the persistent SM-pair kernel below -- a
// cluster of two CTAs owns 256 x 256 output tiles, the leader drives both tensor cores with
// cta_group::2 MMAs, two accumulators in tensor memory let one tile's epilogue overlap the next
// tile's MMAs. Other D (multiples of 128): one CTA per 128 x 128 tile. Either way each tile
// reduces over all n token rows in a fixed order (no atomics: results repeat bit for bit), and
// several layers whose operands lie contiguously ([layers][n][D]) go in one launch, so that a
// warmup chunk's statistics fill the GPU instead of one short wave per layer; each tile's
// arithmetic does not depend on the batching. G and H are symmetric: only tiles on or above
// the block diagonal are computed, and each is written to both mirrored positions, so the
// stored G and H are exactly symmetric.
//
// Both MMA operands are "MN-major" slices of [n, D]: a TMA box of 64 token rows x 64
// columns (128-byte swizzle) puts 64 columns of one token in each 128-byte row, with
// consecutive tokens (the reduction index) 128 bytes apart. 256 threads: warp 0 TMA,
// warp 1 MMA, warps 4..7 epilogue (read-modify-write of the float32 tile).
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;         // output tile rows; column blocks of 128
constexpr int kKRows = 64;         // token rows per stage
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Tiles of 128 x kN outputs: kN = 256 halves the A-operand bytes per flop (2 stages of 48 KB,
// two CTAs per SM); kN = 128 for D not a multiple of 256 (3 stages of 32 KB).
template <int kN>
struct StatsCfg {
    static constexpr int kStages = kN == 256 ? 2 : 3;
    static constexpr int kABytes = kKRows * kTile * 2;           // 16 KB: two 64x64 boxes
    static constexpr int kBBytes = kKRows * kN * 2;              // kN / 64 boxes
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmemAlloc = kBarOff + 256 + 1024;
    static constexpr int kBlocks = kN / kTile;                   // 128-column blocks per tile
};

struct StatsParams {
    float *out[kMaxBatch][3];   // per layer: G, C, H
    int D, n;
    int nb;             // D / 128
    int ng;             // column groups per row: D / kN
    int n_sym;          // tiles per symmetric matrix that touch its upper triangle
    int *err_flag;
};

// Work item -> (matrix, tile row bi, column group g). Items 0..n_sym-1: G, then C (nb*ng),
// then H (n_sym). A symmetric matrix keeps, in row bi, the groups whose last column block
// is on or above the diagonal: g >= bi / kBlocks.
template <int kBlocks>
__device__ __forceinline__ void decode_item(int item, int nb, int ng, int n_sym, int &mat, int &bi, int &g) {
    int t;
    if (item < n_sym) { mat = 0; t = item; }
    else if (item < n_sym + nb * ng) { mat = 1; bi = (item - n_sym) / ng; g = (item - n_sym) % ng; return; }
    else { mat = 2; t = item - n_sym - nb * ng; }
    int r = 0;
    while (t >= ng - r / kBlocks) { t -= ng - r / kBlocks; ++r; }
    bi = r;
    g = r / kBlocks + t;
}

template <int kN>
__global__ void __launch_bounds__(kThreads, 2)
stats_gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmR,
                        const StatsParams p) {
    using Cfg = StatsCfg<kN>;
    constexpr int kStages = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *acc_bar = empty + kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int layer = blockIdx.y;
    int mat, bi, g;
    decode_item<Cfg::kBlocks>(blockIdx.x, p.nb, p.ng, p.n_sym, mat, bi, g);
    const CUtensorMap *mapA = (mat == 2) ? &tmR : &tmA;   // left operand: A for G and C, R for H
    const CUtensorMap *mapB = (mat == 0) ? &tmA : &tmR;   // right operand: A for G, R for C and H
    const int n_k = (p.n + kKRows - 1) / kKRows;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(acc_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, kN);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // producer and MMA warps stay converged; one elected lane issues (uniform registers)
    if (warp == 0) {
        if (lane == 0) {
            ptx::tma_prefetch_desc(mapA);
            ptx::tma_prefetch_desc(mapB);
        }
        const uint64_t pol = ptx::policy_evict_last();
        int issued = -1;
        bool ok = true;
        for (int kt = 0; kt < n_k && ok; ++kt) {
            const int s = kt % kStages;
            const uint32_t ph = (kt / kStages) & 1;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&empty[s], ph ^ 1, kWaitLimitNs, p.err_flag, abort_flag));
            if (!ok) break;
            uint8_t *base = smem + s * Cfg::kStageBytes;
            ptx::mbar_arrive_expect_tx_warp(&full[s], Cfg::kStageBytes);
#pragma unroll
            for (int b = 0; b < 2; ++b)
                ptx::tma_load_3d_warp(base + b * (kKRows * 128), mapA, &full[s], bi * kTile + b * 64, kt * kKRows,
                                      layer, pol);
#pragma unroll
            for (int b = 0; b < kN / 64; ++b)
                ptx::tma_load_3d_warp(base + Cfg::kABytes + b * (kKRows * 128), mapB, &full[s], g * kN + b * 64,
                                      kt * kKRows, layer, pol);
            issued = kt;
        }
        if (!ok) {
            for (int kt = (issued - kStages + 1 > 0 ? issued - kStages + 1 : 0); kt <= issued; ++kt)
                ptx::mbar_wait_bounded(&full[kt % kStages], (kt / kStages) & 1, kWaitLimitNs, nullptr, nullptr);
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc = ptx::make_idesc_bf16(kTile, kN, true, true);
        const uint32_t sbase = ptx::smem_u32(smem);
        bool ok = true;
        for (int kt = 0; kt < n_k && ok; ++kt) {
            const int s = kt % kStages;
            ok = __all_sync(0xffffffffu,
                            ptx::mbar_wait_bounded(&full[s], (kt / kStages) & 1, kWaitLimitNs, p.err_flag, abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t a0 = sbase + s * Cfg::kStageBytes;
            const uint32_t b0 = a0 + Cfg::kABytes;
#pragma unroll
            for (int kk = 0; kk < kKRows / 16; ++kk) {
                // both operands MN-major: 64-column groups kKRows * 128 bytes apart
                const uint64_t da = ptx::make_sdesc_sw128(a0 + kk * 2048, kKRows * 128, 1024);
                const uint64_t db = ptx::make_sdesc_sw128(b0 + kk * 2048, kKRows * 128, 1024);
                ptx::umma_f16_ss_warp(tmem, da, db, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::umma_commit_warp(&empty[s]);
        }
        if (!ok) {
            if (lane == 0) *abort_flag = 1;
            __threadfence_block();
        }
        ptx::umma_commit_warp(acc_bar);
        ptx::mbar_wait_bounded(acc_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
    } else if (warp >= 4) {
        const int wq = warp - 4;
        const int r = wq * 32 + lane;                   // row inside the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const bool ok = ptx::mbar_wait_bounded(acc_bar, 0, kWaitLimitNs, p.err_flag, abort_flag) && !*abort_flag;
        if (ok) {
            ptx::tc_fence_after();
            float *M = p.out[layer][mat];
            const size_t D = p.D;
            const int gi = bi * kTile + r;
            const bool sym = (mat != 1);
#pragma unroll 1
            for (int c = 0; c < kN / 32; ++c) {
                const int gj0 = g * kN + c * 32;
                const int bj = gj0 / kTile;                 // 128-column block of this chunk
                if (sym && bj < bi) continue;               // below the diagonal: the mirror holds it
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_off + c * 32, v);
                ptx::tmem_wait_ld();
                float *rowp = M + (size_t)gi * D + gj0;
                if (!(sym && bj == bi)) {
#pragma unroll
                    for (int q = 0; q < 32; q += 4) {
                        float4 o = *reinterpret_cast<const float4 *>(rowp + q);
                        o.x += __uint_as_float(v[q]);
                        o.y += __uint_as_float(v[q + 1]);
                        o.z += __uint_as_float(v[q + 2]);
                        o.w += __uint_as_float(v[q + 3]);
                        *reinterpret_cast<float4 *>(rowp + q) = o;
                        if (sym) {
                            M[(size_t)(gj0 + q) * D + gi] = o.x;
                            M[(size_t)(gj0 + q + 1) * D + gi] = o.y;
                            M[(size_t)(gj0 + q + 2) * D + gi] = o.z;
                            M[(size_t)(gj0 + q + 3) * D + gi] = o.w;
                        }
                    }
                } else {
                    // diagonal block: the upper triangle (j >= i) is updated and mirrored
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        const int gj = gj0 + q;
                        if (gj >= gi) {
                            const float o = rowp[q] + __uint_as_float(v[q]);
                            rowp[q] = o;
                            if (gj > gi) M[(size_t)gj * D + gi] = o;
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kN);
    }
}

// ---------------------------------------------------------------------------------------
// SM-pair kernel (D a multiple of 256): one cluster of two CTAs on two SMs owns a 256 x 256
// output tile; the leader issues tcgen05.mma.cta_group::2 with M = 256 (each CTA's 128 output
// rows in its own tensor memory) and N = 256 (each CTA holds 128 of the 256 columns of the
// right operand). Per SM and k-step that halves the operand bytes of a 128 x 256 tile per flop
// (64 instead of 96 B/clk read by the tensor core, 64 instead of 96 B/clk written by TMA), which
// keeps shared memory below its 128 B/clk. The kernel is persistent: cluster c takes tiles
// c, c + clusters, ... of all layers in order, with two accumulators of 256 columns in tensor
// memory, so that one tile's read-modify-write epilogue overlaps the next tile's MMAs. Each
// tile still reduces over all n token rows in a fixed order (no atomics).
constexpr int kPairStages = 7;
constexpr int kPairHalf = 128;                              // output rows / right-operand columns per CTA
constexpr int kPairOpBytes = kKRows * kPairHalf * 2;        // 16 KB: two 64 x 64 boxes
constexpr int kPairStageBytes = 2 * kPairOpBytes;           // left + right operand of this CTA
constexpr int kPairOffBar = kPairStages * kPairStageBytes;
constexpr int kPairNumBars = 2 * kPairStages + 2 + 2 + 1;   // full, empty, acc_full[2], acc_empty[2], done
constexpr int kPairSmem = kPairOffBar + kPairNumBars * 8 + 16 + 1024;
static_assert(kPairSmem <= 232448, "shared memory budget");

struct PairParams {
    float *out[kMaxBatch][3];   // per layer: G, C, H
    int D, n;
    int nb;                     // D / 256
    int n_sym;                  // nb (nb + 1) / 2 tiles on or above the block diagonal
    int items;                  // tiles per layer: G, C, H
    int tiles;                  // items * layers
    int *err_flag;
};

// Work item of a layer -> (matrix, tile row bi, tile column g) in 256-blocks: G's upper tiles,
// then every C tile, then H's upper tiles.
__device__ __forceinline__ void decode_pair_item(int item, int nb, int n_sym, int &mat, int &bi, int &g) {
    int t;
    if (item < n_sym) { mat = 0; t = item; }
    else if (item < n_sym + nb * nb) { mat = 1; bi = (item - n_sym) / nb; g = (item - n_sym) % nb; return; }
    else { mat = 2; t = item - n_sym - nb * nb; }
    int r = 0;
    while (t >= nb - r) { t -= nb - r; ++r; }
    bi = r;
    g = r + t;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
stats_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmR,
                  const PairParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    // both CTAs evaluate the same condition, so either both leave here or neither does
    if (ptx::cluster_nctarank() != 2) {
        if (threadIdx.x == 0) raise_device_error(p.err_flag, ISPA_ERR_UNSUPPORTED);
        return;
    }
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kPairOffBar);   // [stages] (leader's count both CTAs)
    uint64_t *empty = full + kPairStages;                                // [stages] (multicast commit)
    uint64_t *acc_full = empty + kPairStages;                            // [2] (multicast commit)
    uint64_t *acc_empty = acc_full + 2;                                  // [2] (leader's: 4 warps x 2 CTAs)
    uint64_t *done_bar = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cl = blockIdx.x / 2, ncl = gridDim.x / 2;
    const int n_k = (p.n + kKRows - 1) / kKRows;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], 8);
        }
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc_2sm(tmem_slot, 512);
        ptx::tmem_relinquish_2sm();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();      // the peer's barriers exist before anything arrives on them
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmA);
            ptx::tma_prefetch_desc(&tmR);
        }
        const uint64_t pol = ptx::policy_evict_last();
        int it = 0;
        bool ok = true;
        for (int t = cl; t < p.tiles && ok; t += ncl) {
            const int layer = t / p.items;
            int mat, bi, g;
            decode_pair_item(t % p.items, p.nb, p.n_sym, mat, bi, g);
            const CUtensorMap *mapL = (mat == 2) ? &tmR : &tmA;   // left operand: A for G and C, R for H
            const CUtensorMap *mapR = (mat == 0) ? &tmA : &tmR;   // right operand: A for G, R for C and H
            const int rowL = bi * 256 + (int)rank * kPairHalf;
            const int colR = g * 256 + (int)rank * kPairHalf;
            for (int kt = 0; kt < n_k; ++kt, ++it) {
                const int s = it % kPairStages;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded_cluster(&empty[s], ((it / kPairStages) & 1) ^ 1,
                                                                            kWaitLimitNs, p.err_flag, abort_flag));
                if (!ok) break;
                uint8_t *base = smem + s * kPairStageBytes;
                const uint32_t lead_full = ptx::mapa_shared(ptx::smem_u32(&full[s]), 0);
                if (leader) ptx::mbar_arrive_expect_tx_warp(&full[s], 2 * kPairStageBytes);
                if (ptx::elect_one()) {
#pragma unroll
                    for (int b = 0; b < 2; ++b)
                        ptx::tma_load_3d_2sm(base + b * (kKRows * 128), mapL, lead_full, rowL + b * 64, kt * kKRows,
                                             layer, pol);
#pragma unroll
                    for (int b = 0; b < 2; ++b)
                        ptx::tma_load_3d_2sm(base + kPairOpBytes + b * (kKRows * 128), mapR, lead_full, colR + b * 64,
                                             kt * kKRows, layer, pol);
                }
                __syncwarp();
            }
        }
        if (!ok) {
            // let copies in flight land before the CTA can exit (bounded)
            const uint64_t t0 = ptx::globaltimer_ns();
            while (ptx::globaltimer_ns() - t0 < 2000000ull) {
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader) {
            constexpr uint32_t idesc = ptx::make_idesc_bf16(2 * kPairHalf, 256, true, true);
            const uint32_t sbase = ptx::smem_u32(smem);
            int it = 0, i = 0;
            bool ok = true;
            for (int t = cl; t < p.tiles && ok; t += ncl, ++i) {
                const int b = i & 1;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded_cluster(&acc_empty[b], ((i >> 1) & 1) ^ 1,
                                                                            kWaitLimitNs, p.err_flag, abort_flag));
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)b * 256u;
                for (int kt = 0; kt < n_k; ++kt, ++it) {
                    const int s = it % kPairStages;
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded_cluster(&full[s], (it / kPairStages) & 1,
                                                                                kWaitLimitNs, p.err_flag, abort_flag));
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint32_t a0 = sbase + s * kPairStageBytes;
                    const uint32_t b0 = a0 + kPairOpBytes;
                    if (ptx::elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kKRows / 16; ++kk) {
                            // both operands MN-major: 64-column groups kKRows * 128 bytes apart
                            const uint64_t da = ptx::make_sdesc_sw128(a0 + kk * 2048, kKRows * 128, 1024);
                            const uint64_t db = ptx::make_sdesc_sw128(b0 + kk * 2048, kKRows * 128, 1024);
                            ptx::umma_f16_ss_2sm(d, da, db, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                        }
                        ptx::umma_commit_2sm(&empty[s], 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (ptx::elect_one()) ptx::umma_commit_2sm(&acc_full[b], 0x3);
                __syncwarp();
            }
            if (!ok && lane == 0) *abort_flag = 1;
            // every MMA this CTA issued has completed before the pair releases tensor memory
            if (ptx::elect_one()) ptx::umma_commit_2sm(done_bar, 0x1);
            __syncwarp();
            ptx::mbar_wait_bounded_cluster(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int wq = warp - 4;                           // TMEM lane quarter: rows wq*32 .. +31 of this CTA's half
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t lead_empty0 = ptx::mapa_shared(ptx::smem_u32(&acc_empty[0]), 0);
        const uint32_t lead_empty1 = ptx::mapa_shared(ptx::smem_u32(&acc_empty[1]), 0);
        const size_t D = p.D;
        int i = 0;
        for (int t = cl; t < p.tiles; t += ncl, ++i) {
            const int b = i & 1;
            const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded_cluster(&acc_full[b], (i >> 1) & 1,
                                                                                   kWaitLimitNs, p.err_flag,
                                                                                   abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            const int layer = t / p.items;
            int mat, bi, g;
            decode_pair_item(t % p.items, p.nb, p.n_sym, mat, bi, g);
            float *M = p.out[layer][mat];
            const int warp_row0 = bi * 256 + (int)rank * kPairHalf + wq * 32;
            const int gi = warp_row0 + lane;
            const bool sym = mat != 1;
            const bool diag = sym && bi == g;
            // two 32-column chunks at a time: both chunks' accumulator values and stored values are
            // loaded before either is used, so their memory latencies overlap
#pragma unroll 1
            for (int c2 = 0; c2 < 256 / 64; ++c2) {
                const int gc0 = g * 256 + c2 * 64;
                // warp-uniform: a 32 x 32 block wholly below the diagonal of a symmetric matrix is
                // the mirror of one above it
                const bool skip0 = diag && gc0 + 31 < warp_row0;
                const bool skip1 = diag && gc0 + 63 < warp_row0;
                if (skip0 && skip1) continue;
                uint32_t v[2][32];
                ptx::tmem_ld32(tmem + (uint32_t)b * 256u + lane_off + c2 * 64, v[0]);
                ptx::tmem_ld32(tmem + (uint32_t)b * 256u + lane_off + c2 * 64 + 32, v[1]);
                ptx::tmem_wait_ld();
                float *rowp = M + (size_t)gi * D + gc0;
                const bool full0 = !diag || gc0 > warp_row0 + 31;
                const bool full1 = !diag || gc0 + 32 > warp_row0 + 31;
                float4 old[2][8];
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if ((h == 0 ? full0 : full1))
#pragma unroll
                        for (int q = 0; q < 8; ++q) old[h][q] = *reinterpret_cast<const float4 *>(rowp + 32 * h + 4 * q);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (h == 0 ? skip0 : skip1) continue;
                    const int gj0 = gc0 + 32 * h;
                    float *rp = rowp + 32 * h;
                    if (h == 0 ? full0 : full1) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 o = old[h][q];
                            o.x += __uint_as_float(v[h][4 * q]);
                            o.y += __uint_as_float(v[h][4 * q + 1]);
                            o.z += __uint_as_float(v[h][4 * q + 2]);
                            o.w += __uint_as_float(v[h][4 * q + 3]);
                            *reinterpret_cast<float4 *>(rp + 4 * q) = o;
                            if (sym) {
                                M[(size_t)(gj0 + 4 * q) * D + gi] = o.x;
                                M[(size_t)(gj0 + 4 * q + 1) * D + gi] = o.y;
                                M[(size_t)(gj0 + 4 * q + 2) * D + gi] = o.z;
                                M[(size_t)(gj0 + 4 * q + 3) * D + gi] = o.w;
                            }
                        }
                    } else {
                        // a block on the diagonal: the upper triangle (j >= i) is updated and mirrored
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const int gj = gj0 + q;
                            if (gj >= gi) {
                                const float o = rp[q] + __uint_as_float(v[h][q]);
                                rp[q] = o;
                                if (gj > gi) M[(size_t)gj * D + gi] = o;
                            }
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(b ? lead_empty1 : lead_empty0);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_2sm(tmem, 512);
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

// [layers, n, D] bf16 row-major, box = 64 rows x 64 columns of one layer, 128-byte swizzle.
bool make_panel_map(CUtensorMap *m, const void *ptr, int layers, int n, int D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n, (cuuint64_t)layers};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)n * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kKRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

template <int kN>
cudaError_t launch_tiles(const CUtensorMap &ma, const CUtensorMap &mr, StatsParams p, int layers, cudaStream_t s) {
    using Cfg = StatsCfg<kN>;
    p.ng = p.D / kN;
    p.n_sym = 0;
    for (int bi = 0; bi < p.nb; ++bi) p.n_sym += p.ng - bi / Cfg::kBlocks;
    cudaError_t e = cudaFuncSetAttribute(stats_gemm_sm100_kernel<kN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::kSmemAlloc);
    if (e != cudaSuccess) return e;
    const int items = 2 * p.n_sym + p.nb * p.ng;
    stats_gemm_sm100_kernel<kN><<<dim3(items, layers), kThreads, Cfg::kSmemAlloc, s>>>(ma, mr, p); note_launch();
    return cudaGetLastError();
}

// Persistent SM-pair launch: as many clusters as can be resident (at most one per tile).
cudaError_t launch_pairs(const CUtensorMap &ma, const CUtensorMap &mr, const StatsParams &sp, int layers,
                         cudaStream_t s) {
    PairParams p;
    for (int l = 0; l < layers; ++l)
        for (int m = 0; m < 3; ++m) p.out[l][m] = sp.out[l][m];
    p.D = sp.D;
    p.n = sp.n;
    p.nb = sp.D / 256;
    p.n_sym = p.nb * (p.nb + 1) / 2;
    p.items = 2 * p.n_sym + p.nb * p.nb;
    p.tiles = p.items * layers;
    p.err_flag = sp.err_flag;
    cudaError_t e = cudaFuncSetAttribute(stats_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static int max_clusters[64] = {0};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (max_clusters[dev] <= 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kPairSmem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, stats_pair_kernel, &cfg);
        if (e != cudaSuccess) return e;
        if (n <= 0) return cudaErrorInvalidConfiguration;
        max_clusters[dev] = n;
    }
    const int clusters = p.tiles < max_clusters[dev] ? p.tiles : max_clusters[dev];
    stats_pair_kernel<<<2 * clusters, kThreads, kPairSmem, s>>>(ma, mr, p);
    note_launch();
    return cudaGetLastError();
}

// Layers [0, layers) with operands a_loc, r = [layers][n][D] contiguous and outputs
// G[l], C[l], H[l]; layers <= kMaxBatch.
cudaError_t launch_stats_bf16_layers(const void *a_loc, const void *r, int layers, int n, int D, float *const *G,
                                     float *const *C, float *const *H, int *err_flag, cudaStream_t s) {
    if (n <= 0 || layers <= 0) return cudaSuccess;
    if (layers > kMaxBatch) return cudaErrorInvalidValue;
    if (D % kTile != 0) {
        // D not a multiple of 128 (e.g. 64-wide single head): CUDA-core GEMM, layer by layer
        for (int l = 0; l < layers; ++l) {
            const size_t off = (size_t)l * n * D * sizeof(bf16);
            const void *al = static_cast<const char *>(a_loc) + off;
            const void *rl = static_cast<const char *>(r) + off;
            GemmDesc g{D, D, n, D, D, D, false, false, ElemType::BF16, ElemType::BF16, ElemType::F32, 1.f, 1.f, false, 1};
            GemmBatch b;
            b.A[0] = al; b.B[0] = al; b.C[0] = G[l];
            cudaError_t e = launch_gemm_simt(g, b, s);
            if (e != cudaSuccess) return e;
            b.A[0] = al; b.B[0] = rl; b.C[0] = C[l];
            e = launch_gemm_simt(g, b, s);
            if (e != cudaSuccess) return e;
            b.A[0] = rl; b.B[0] = rl; b.C[0] = H[l];
            e = launch_gemm_simt(g, b, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    CUtensorMap ma, mr;
    if (!make_panel_map(&ma, a_loc, layers, n, D) || !make_panel_map(&mr, r, layers, n, D)) return cudaErrorInvalidValue;
    StatsParams p;
    for (int l = 0; l < layers; ++l) {
        p.out[l][0] = G[l]; p.out[l][1] = C[l]; p.out[l][2] = H[l];
    }
    p.D = D; p.n = n;
    p.nb = D / kTile;
    p.err_flag = err_flag;
    if (D % 256 == 0) return launch_pairs(ma, mr, p, layers, s);
    return launch_tiles<128>(ma, mr, p, layers, s);
}

cudaError_t launch_stats_bf16(const void *a_loc, const void *r, int n, int D, float *G, float *C, float *H,
                              int *err_flag, cudaStream_t s) {
    return launch_stats_bf16_layers(a_loc, r, 1, n, D, &G, &C, &H, err_flag, s);
}

}  // namespace ispa
