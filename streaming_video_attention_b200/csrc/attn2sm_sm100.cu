// Split (decomposable) attention for head_dim 128 on CTA pairs: tcgen05 cta_group::2
// [ISPA §3.1 step 1 "Dual-Stream Warmup", §3.4 "Decomposable Attention"].
//
// Same computation as the single-CTA kernel (two online-softmax states per query row, one per
// KV partition, merged by log-sum-exp in the epilogue; the statistics operands A_loc and R
// written for the Gram GEMM), but two CTAs -- two 128-row query tiles of the same head on two
// SMs -- share every K/V tile:
//   S = Q K^T  : one 256 x 128 x 16 MMA per k-step covers both query tiles; each CTA holds its
//                own Q tile and 64 of the 128 keys of the K tile (the B operand is split by N).
//   O += P V   : A = P from each CTA's own tensor memory; each CTA holds V for 64 of the 128
//                head dimensions (again split by N).
// So each SM loads half of every K/V tile (half the L2 -> SM traffic of the single-CTA
// kernel) and the leader CTA's single MMA thread drives both tensor cores (half the MMA
// issue work per SM). Each CTA still runs its own softmax warps and epilogue on its own 128
// rows and TMEM lanes.
//
// Synchronisation across the pair: both CTAs' TMA loads count on the leader's barriers (its
// producer expects the bytes of both halves); the leader's MMA commits arrive on the barriers
// of both CTAs (multicast commit); the softmax warps of both CTAs arrive on the leader's
// P-ready barrier through cluster addresses. A cluster barrier keeps both CTAs (their shared
// memory and tensor memory) alive until every MMA of the pair has finished. Every mbarrier
// wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int HD = 128;
constexpr int kBlockM = 128;     // query rows per CTA
constexpr int kBlockN = 128;     // KV rows per tile
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int NS = 5;            // K/V stages
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;

constexpr int kQBytes = kBlockM * HD * 2;              // 32 KB
constexpr int kKHalfBytes = (kBlockN / 2) * HD * 2;    // 16 KB: 64 keys x 128 dims
constexpr int kVHalfBytes = kBlockN * (HD / 2) * 2;    // 16 KB: 128 keys x 64 dims
constexpr int kStageBytes = kKHalfBytes + kVHalfBytes;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffBar = kOffKV + NS * kStageBytes;
constexpr int kNumBars = 1 + 2 * NS + 2 + 2 + 1 + 1;
constexpr int kOffSeg = kOffBar + kNumBars * 8;
constexpr int kOffMisc = kOffSeg + 4 * kMaxSegments * 4;
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmem = kSmemUsed + 1024;   // slack for aligning the base to the 128-byte swizzle atom
static_assert(kSmem <= 232448, "shared memory budget");

struct Split2Params {
    void *o_full;
    float *lse_full;
    void *o_loc;
    float *lse_loc;
    void *o_hist;
    float *lse_hist;
    void *a_ops;
    void *r_ops;
    int n_q, heads;
    float scale_log2;
    SegmentList segs;
    int *err_flag;
};

struct TileCursor {
    const int *sb, *se, *sp, *sf;
    int nseg, si, row0, end, part, seg_first, tile_in_seg;
    __device__ __forceinline__ void init(const int *b, const int *e, const int *pt, const int *f, int n) {
        sb = b; se = e; sp = pt; sf = f; nseg = n; si = 0;
        if (n > 0) load();
    }
    __device__ __forceinline__ void load() {
        row0 = sb[si]; end = se[si]; part = sp[si]; seg_first = sf[si]; tile_in_seg = 0;
    }
    __device__ __forceinline__ void advance() {
        row0 += kBlockN;
        ++tile_in_seg;
        if (row0 >= end && ++si < nseg) load();
    }
    __device__ __forceinline__ int valid() const { return min(kBlockN, end - row0); }
    __device__ __forceinline__ bool first_of_part() const { return seg_first && tile_in_seg == 0; }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_split_2sm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK64,
                      const __grid_constant__ CUtensorMap tmV, const Split2Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    // both CTAs evaluate the same condition, so either both leave here or neither does
    if (ptx::cluster_nctarank() != 2) {
        if (threadIdx.x == 0) atomicCAS(p.err_flag, 0, ISPA_ERR_UNSUPPORTED);
        return;
    }
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    uint8_t *sQ = smem + kOffQ;
    uint8_t *sKV = smem + kOffKV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *q_full = bars;
    uint64_t *kv_full = q_full + 1;       // [NS] (leader's counts the bytes of both CTAs)
    uint64_t *kv_empty = kv_full + NS;    // [NS] (multicast commit after the tile's PV)
    uint64_t *s_full = kv_empty + NS;     // [2]
    uint64_t *p_full = s_full + 2;        // [2]  (leader's: 4 softmax warps x 2 CTAs)
    uint64_t *o_bar = p_full + 2;
    uint64_t *done_bar = o_bar + 1;
    int *seg_begin = reinterpret_cast<int *>(smem + kOffSeg);
    int *seg_end = seg_begin + kMaxSegments;
    int *seg_part = seg_end + kMaxSegments;
    int *seg_first = seg_part + kMaxSegments;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int q0 = blockIdx.x * kBlockM;
    const int head = blockIdx.y;
    const int nseg = p.segs.count;
    int n_tiles = 0;
    for (int s = 0; s < nseg; ++s) n_tiles += (p.segs.seg[s].end - p.segs.seg[s].begin + kBlockN - 1) / kBlockN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nseg; ++s) {
            const Segment sg = p.segs.seg[s];
            seg_begin[s] = sg.begin;
            seg_end[s] = sg.end;
            seg_part[s] = sg.part;
            int first = 1;
            for (int u = 0; u < s; ++u)
                if (p.segs.seg[u].part == sg.part) first = 0;
            seg_first[s] = first;
        }
        ptx::mbar_init(q_full, 1);
        for (int i = 0; i < NS; ++i) {
            ptx::mbar_init(&kv_full[i], 1);
            ptx::mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s_full[i], 1);
            ptx::mbar_init(&p_full[i], 8);
        }
        ptx::mbar_init(o_bar, 1);
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
    auto tS = [tmem](int st) { return tmem + (uint32_t)st * 128u; };
    auto tO = [tmem](int q) { return tmem + 256u + (uint32_t)q * (uint32_t)HD; };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmQ);
            ptx::tma_prefetch_desc(&tmK64);
            ptx::tma_prefetch_desc(&tmV);
            const uint64_t pol_q = ptx::policy_evict_first();
            const uint64_t pol_kv = ptx::policy_evict_last();
            const uint32_t lead_q_full = ptx::mapa_shared(ptx::smem_u32(q_full), 0);
            if (leader) ptx::mbar_arrive_expect_tx(q_full, 2 * kQBytes);
            for (int b = 0; b < HD / 64; ++b)
                ptx::tma_load_3d_2sm(sQ + b * (kBlockM * 128), &tmQ, lead_q_full, b * 64, head, q0, pol_q);
            TileCursor cur;
            cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
            bool ok = true;
            for (int j = 0; j < n_tiles; ++j, cur.advance()) {
                const int st = j % NS;
                ok = ptx::mbar_wait_bounded_cluster(&kv_empty[st], ((j / NS) & 1) ^ 1, kWaitLimitNs, p.err_flag, abort_flag);
                if (!ok) break;
                uint8_t *sK = sKV + st * kStageBytes;
                uint8_t *sV = sK + kKHalfBytes;
                const uint32_t lead_full = ptx::mapa_shared(ptx::smem_u32(&kv_full[st]), 0);
                if (leader) ptx::mbar_arrive_expect_tx(&kv_full[st], 2 * kStageBytes);
                // keys row0 + 64*rank .. +63, all 128 dims (two 64-dim boxes)
                for (int b = 0; b < HD / 64; ++b)
                    ptx::tma_load_3d_2sm(sK + b * ((kBlockN / 2) * 128), &tmK64, lead_full, b * 64, head,
                                         cur.row0 + 64 * (int)rank, pol_kv);
                // all 128 keys, dims 64*rank .. +63
                ptx::tma_load_3d_2sm(sV, &tmV, lead_full, 64 * (int)rank, head, cur.row0, pol_kv);
            }
            if (!ok) {
                // let copies in flight land before the CTA can exit (bounded)
                const uint64_t t0 = ptx::globaltimer_ns();
                while (ptx::globaltimer_ns() - t0 < 2000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc_qk = ptx::make_idesc_bf16(2 * kBlockM, kBlockN, false, false);
            constexpr uint32_t idesc_pv = ptx::make_idesc_bf16(2 * kBlockM, HD, false, true);
            const uint32_t aQ = ptx::smem_u32(sQ), aKV = ptx::smem_u32(sKV);
            bool ok = ptx::mbar_wait_bounded_cluster(q_full, 0, kWaitLimitNs, p.err_flag, abort_flag);
            auto issue_s = [&](int j) -> bool {
                const int sb = j & 1, ks = j % NS;
                if (!ptx::mbar_wait_bounded_cluster(&kv_full[ks], (j / NS) & 1, kWaitLimitNs, p.err_flag, abort_flag))
                    return false;
                ptx::tc_fence_after();
                const uint32_t aK = aKV + ks * kStageBytes;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t da = ptx::make_sdesc_sw128(aQ + (kk / 4) * (kBlockM * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t db =
                        ptx::make_sdesc_sw128(aK + (kk / 4) * ((kBlockN / 2) * 128) + (kk % 4) * 32, 16, 1024);
                    ptx::umma_f16_ss_2sm(tS(sb), da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::umma_commit_2sm(&s_full[sb], 0x3);
                return true;
            };
            if (ok && n_tiles > 0) ok = issue_s(0);
            TileCursor cur;
            cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
            for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
                if (j + 1 < n_tiles) {
                    ok = issue_s(j + 1);
                    if (!ok) break;
                }
                const int sb = j & 1, vs = j % NS;
                const uint32_t acc0 = cur.first_of_part() ? 0u : 1u;
                const uint32_t dO = tO(cur.part);
                ok = ptx::mbar_wait_bounded_cluster(&p_full[sb], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t aV = aKV + vs * kStageBytes + kKHalfBytes;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint64_t db = ptx::make_sdesc_sw128(aV + kk * 2048, kBlockN * 128, 1024);
                    ptx::umma_f16_ts_2sm(dO, tS(sb) + kk * 8, db, idesc_pv, kk > 0 ? 1u : acc0);
                }
                ptx::umma_commit_2sm(o_bar, 0x3);
                ptx::umma_commit_2sm(&kv_empty[vs], 0x3);
            }
            ptx::umma_commit_2sm(done_bar, 0x1);
            ptx::mbar_wait_bounded_cluster(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------------ softmax + epilogue (both CTAs)
        const int wq = warp - kSoftmaxWarp0;
        const int row = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        float m_loc = -INFINITY, m_hist = -INFINITY;
        float l_loc = 0.f, l_hist = 0.f;
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        const uint32_t lead_p_full0 = ptx::mapa_shared(ptx::smem_u32(&p_full[0]), 0);
        const uint32_t lead_p_full1 = ptx::mapa_shared(ptx::smem_u32(&p_full[1]), 0);
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
            const int st = j & 1;
            const int valid = cur.valid();
            const int part = cur.part;
            ok = ptx::mbar_wait_bounded_cluster(&s_full[st], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            uint32_t sr[kBlockN];
#pragma unroll
            for (int c = 0; c < kBlockN / 32; ++c)
                ptx::tmem_ld32(tS(st) + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            ptx::tmem_wait_ld();
            float *s = reinterpret_cast<float *>(sr);
            if (valid < kBlockN) {
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int c = 4; c < kBlockN; c += 8) {
#pragma unroll
                for (int u = 0; u < 4; ++u) mx4[u] = ptx::max3(mx4[u], s[c + u], s[c + 4 + u < kBlockN ? c + 4 + u : c + u]);
            }
            float mx = ptx::max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
            mx *= p.scale_log2;
            float m_cur = part ? m_hist : m_loc;
            float l_cur = part ? l_hist : l_loc;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_cur + kRescaleThreshold || m_cur == -INFINITY) {
                if (m_cur != -INFINITY) {
                    alpha = exp2f(m_cur - mx);
                    rescale = true;
                }
                m_cur = mx;
            }
            float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[kBlockN / 2];
            const float neg_m = -m_cur;
#pragma unroll
            for (int c = 0; c < kBlockN; c += 2) {
                const float e0 = ptx::exp2_approx(fmaf(s[c], p.scale_log2, neg_m));
                const float x1 = fmaf(s[c + 1], p.scale_log2, neg_m);
                const float e1 = ((c / 2) % 2 == 1) ? ptx::exp2_poly(x1) : ptx::exp2_approx(x1);
                sum8[(c / 2) % 8] += e0 + e1;
                pk[c / 2] = pack_bf16x2(e0, e1);
            }
            const float rowsum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            l_cur = fmaf(l_cur, alpha, rowsum);
            if (part) { m_hist = m_cur; l_hist = l_cur; } else { m_loc = m_cur; l_loc = l_cur; }
            ptx::tmem_st32(tS(st) + lane_off, &pk[0]);
            ptx::tmem_st32(tS(st) + lane_off + 32, &pk[32]);
            ptx::tmem_wait_st();
            // O may be rescaled only once PV_{j-1} is complete. Without a rescale there is nothing
            // to wait for: PV_j queues behind PV_{j-1} on the tensor pipe, and P_j's buffer was
            // last read by PV_{j-2}, which completed before S_j (s_full tracks every earlier MMA).
            // The same fact keeps the o_bar phase here at j-1 or j, so the parity wait is exact.
            // The last tile always waits, so that the epilogue's wait (phase n-1) is exact too.
            const bool rescale_warp = __any_sync(0xffffffffu, rescale);
            if ((rescale_warp || j == n_tiles - 1) && j >= 1) {
                ok = ptx::mbar_wait_bounded_cluster(o_bar, (j - 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
                if (!ok) break;
            }
            if (rescale_warp) {
                ptx::tc_fence_after();
#pragma unroll
                for (int c = 0; c < HD / 16; ++c) {
                    uint32_t r[16];
                    ptx::tmem_ld16(tO(part) + lane_off + c * 16, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    ptx::tmem_st16(tO(part) + lane_off + c * 16, r);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(st ? lead_p_full1 : lead_p_full0);
        }
        // ---------------------------------------------------------------- epilogue
        if (ok && n_tiles > 0) ok = ptx::mbar_wait_bounded_cluster(o_bar, (n_tiles - 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
        if (ok) {
            ptx::tc_fence_after();
            const int qrow = q0 + row;
            const bool active = qrow < p.n_q;
            constexpr float kLn2 = 0.69314718055994530942f;
            const float L2l = l_loc > 0.f ? m_loc + log2f(l_loc) : -INFINITY;
            const float L2h = l_hist > 0.f ? m_hist + log2f(l_hist) : -INFINITY;
            const float mx = fmaxf(L2l, L2h);
            float w_loc = 0.f, w_hist = 0.f, lse_full = -INFINITY;
            if (mx != -INFINITY) {
                const float el = exp2f(L2l - mx), eh = exp2f(L2h - mx);
                w_loc = el / (el + eh);
                w_hist = eh / (el + eh);
                lse_full = (mx + log2f(el + eh)) * kLn2;
            }
            const float inv_l0 = l_loc > 0.f ? 1.f / l_loc : 0.f, inv_l1 = l_hist > 0.f ? 1.f / l_hist : 0.f;
            const bool has0 = l_loc > 0.f, has1 = l_hist > 0.f;
            const size_t D = (size_t)p.heads * HD;
            const size_t obase = ((size_t)qrow * p.heads + head) * HD;
            const size_t sbase = (size_t)qrow * D + (size_t)head * HD;
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t rl[32], rh[32];
                ptx::tmem_ld32(tO(0) + lane_off + c * 32, rl);
                ptx::tmem_ld32(tO(1) + lane_off + c * 32, rh);
                ptx::tmem_wait_ld();
                if (!active) continue;
                uint32_t of[16], ol[16], oh[16], orr[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float al0 = has0 ? __uint_as_float(rl[i]) * inv_l0 : 0.f;
                    const float al1 = has0 ? __uint_as_float(rl[i + 1]) * inv_l0 : 0.f;
                    const float ah0 = has1 ? __uint_as_float(rh[i]) * inv_l1 : 0.f;
                    const float ah1 = has1 ? __uint_as_float(rh[i + 1]) * inv_l1 : 0.f;
                    of[i / 2] = pack_bf16x2(w_loc * al0 + w_hist * ah0, w_loc * al1 + w_hist * ah1);
                    ol[i / 2] = pack_bf16x2(al0, al1);
                    oh[i / 2] = pack_bf16x2(ah0, ah1);
                    orr[i / 2] = pack_bf16x2(w_hist * (ah0 - al0), w_hist * (ah1 - al1));
                }
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<bf16 *>(p.o_full) + obase + c * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) dst[v] = make_uint4(of[4 * v], of[4 * v + 1], of[4 * v + 2], of[4 * v + 3]);
                if (p.o_loc) {
                    uint4 *d2 = reinterpret_cast<uint4 *>(static_cast<bf16 *>(p.o_loc) + obase + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) d2[v] = make_uint4(ol[4 * v], ol[4 * v + 1], ol[4 * v + 2], ol[4 * v + 3]);
                }
                if (p.o_hist) {
                    uint4 *d3 = reinterpret_cast<uint4 *>(static_cast<bf16 *>(p.o_hist) + obase + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) d3[v] = make_uint4(oh[4 * v], oh[4 * v + 1], oh[4 * v + 2], oh[4 * v + 3]);
                }
                if (p.a_ops) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(static_cast<bf16 *>(p.a_ops) + sbase + c * 32);
                    uint4 *d5 = reinterpret_cast<uint4 *>(static_cast<bf16 *>(p.r_ops) + sbase + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        d4[v] = make_uint4(ol[4 * v], ol[4 * v + 1], ol[4 * v + 2], ol[4 * v + 3]);
                        d5[v] = make_uint4(orr[4 * v], orr[4 * v + 1], orr[4 * v + 2], orr[4 * v + 3]);
                    }
                }
            }
            if (active) {
                const size_t li = (size_t)head * p.n_q + qrow;
                p.lse_full[li] = lse_full;
                if (p.lse_loc) p.lse_loc[li] = L2l == -INFINITY ? -INFINITY : L2l * kLn2;
                if (p.lse_hist) p.lse_hist[li] = L2h == -INFINITY ? -INFINITY : L2h * kLn2;
            }
        }
    }

    // every MMA of the pair has finished (the leader waited for them) before either CTA
    // releases tensor memory or leaves
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

// [rows, heads, 128] bf16, box = box_rows rows x 64 dims of one head, 128-byte swizzle.
bool make_rows_map(CUtensorMap *m, const void *ptr, int rows, int heads, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)heads * HD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// head_dim 128 only. The grid's query-tile count is rounded up to even (a tile past n_q
// computes on zero-filled rows and stores nothing).
cudaError_t launch_attn_bf16_2sm(const AttnArgs &a, cudaStream_t s) {
    if (a.n_q == 0) return cudaSuccess;
    if (a.head_dim != HD) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    const void *kp = a.n_kv > 0 ? a.k : a.q;
    const void *vp = a.n_kv > 0 ? a.v : a.q;
    const int kv_rows = a.n_kv > 0 ? a.n_kv : a.n_q;
    if (!make_rows_map(&mq, a.q, a.n_q, a.heads, kBlockM) || !make_rows_map(&mk, kp, kv_rows, a.heads, kBlockN / 2) ||
        !make_rows_map(&mv, vp, kv_rows, a.heads, kBlockN))
        return cudaErrorInvalidValue;
    Split2Params p;
    p.o_full = a.o_full; p.lse_full = a.lse_full;
    p.o_loc = a.o_loc; p.lse_loc = a.lse_loc;
    p.o_hist = a.o_hist; p.lse_hist = a.lse_hist;
    p.a_ops = a.a_loc_ops; p.r_ops = a.r_ops;
    p.n_q = a.n_q; p.heads = a.heads;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.segs = a.segs;
    p.err_flag = a.err_flag;
    cudaError_t e = cudaFuncSetAttribute(attn_split_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const int qt = (a.n_q + kBlockM - 1) / kBlockM;
    dim3 grid((qt + 1) / 2 * 2, a.heads);
    attn_split_2sm_kernel<<<grid, kThreads, kSmem, s>>>(mq, mk, mv, p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace ispa
