// Split (decomposable) attention on the sm_100a tensor cores, bf16 operands, float32
// softmax and accumulation [ISPA §3.1 step 1 "Dual-Stream Warmup", §3.4 "Decomposable
// Attention"].
//
// One pass over the KV rows of one layer keeps two online-softmax states per query row:
// the local partition (sink frame + current chunk) and the history partition (all other
// rows). Each partition has its own float32 accumulator in tensor memory; the epilogue
// merges them by their log-sum-exps into the full output, so the full and the local
// attention cost one attention pass. The epilogue also forms the statistics operands
// A_loc and R = A_full - A_loc = w_hist (A_hist - A_loc) in registers and stores them
// (bf16) for the statistics GEMM that follows on the same stream.
//
// CTA = one 128-row query tile of one head; 256 threads:
//   warp 0      TMA producer: Q once, then K and V tiles of 128 rows into a ring of stages
//   warp 1      TMEM allocation; lane 0 issues every tcgen05.mma and commit
//   warps 4..7  softmax (thread i owns query row i = TMEM lane i), lazy rescale, epilogue
// TMEM (512 columns): S double buffer (2 x 128), O_loc (HD), O_hist (HD). P (bf16) is
// written over the first 64 columns of the S buffer it came from and feeds the PV MMA
// straight from tensor memory; shared memory holds only Q and the K/V ring (TMA, 128-byte
// swizzle).
//
// MMA order S_0, S_1, PV_0, S_2, PV_1, ...: S_{j+1} runs on the tensor cores while the
// softmax works on S_j. tcgen05.mma operations execute in issue order, so S_{j+2} (which
// overwrites S buffer j%2, holding P_j) starts only after PV_j has consumed P_j, and the
// completion of S_j implies that of PV_{j-2}. The MMA thread keeps its non-issuing work per
// tile to two barrier waits and a few integer updates: the tensor-core queue is shallow,
// and every cycle it spends elsewhere is idle tensor time.
//
// The running maximum is updated lazily: a row's reference maximum moves (and its O
// accumulator is rescaled through TMEM) only when a new tile's maximum exceeds it by more
// than 2^8; otherwise exponentials are taken against the stale maximum (values <= 256).
// Output and log-sum-exp stay exact because O and l always share the same reference.
//
// Every mbarrier wait is bounded: on timeout the CTA records ISPA_ERR_TIMEOUT in the
// device flag, every role leaves its loop, outstanding copies and MMAs are awaited (also
// bounded) and TMEM is released before the CTA exits.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int kBlockM = 128;   // query rows per CTA
constexpr int kBlockN = 128;   // KV rows per tile
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;          // log2 units: rescale when the max grows by > 2^8

template <int HD>
struct Smem {
    static constexpr int kStages = HD == 128 ? 3 : 4;   // K/V ring depth
    static constexpr int kQBytes = kBlockM * HD * 2;
    static constexpr int kKVBytes = kBlockN * HD * 2;    // one of K or V for one tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;
    static constexpr int kV = kK + kStages * kKVBytes;
    static constexpr int kBar = kV + kStages * kKVBytes;
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2;   // q, kv full/empty, s_full, p_full, o, done
    static constexpr int kSeg = kBar + kNumBars * 8;              // segment table: 4 x kMaxSegments ints
    static constexpr int kMisc = kSeg + 4 * kMaxSegments * 4;
    static constexpr int kTotal = kMisc + 16;
    static constexpr int kAlloc = kTotal + 1024;   // slack for 1024-byte alignment
};

struct SplitParams {
    void *o_full;
    float *lse_full;
    void *o_loc;
    float *lse_loc;
    void *o_hist;
    float *lse_hist;
    void *a_ops;
    void *r_ops;
    int n_q, heads;
    float scale_log2;   // softmax scale * log2(e)
    SegmentList segs;
    int *err_flag;
};

// Walks the KV tiles in order: the local segments, then the history segments, 128 rows at
// a time (the last tile of a segment may be partial). Segment data sit in shared memory;
// the current segment's bounds stay in registers, so advancing costs an add and a compare.
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
    // first tile of its partition: the accumulator starts from zero
    __device__ __forceinline__ bool first_of_part() const { return seg_first && tile_in_seg == 0; }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
attn_split_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const SplitParams p) {
    using L = Smem<HD>;
    constexpr int NS = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::kQ;
    uint8_t *sK = smem + L::kK;
    uint8_t *sV = smem + L::kV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *q_full = bars + 0;
    uint64_t *kv_full = bars + 1;             // [NS] K and V of one tile landed
    uint64_t *kv_empty = kv_full + NS;        // [NS] S and PV of that tile done
    uint64_t *s_full = kv_empty + NS;         // [2]  S buffer written by the MMA
    uint64_t *p_full = s_full + 2;            // [2]  P written (and O rescaled) by the softmax
    uint64_t *o_bar = p_full + 2;             //      one phase per PV
    uint64_t *done_bar = o_bar + 1;           //      every MMA of this CTA finished
    int *seg_begin = reinterpret_cast<int *>(smem + L::kSeg);
    int *seg_end = seg_begin + kMaxSegments;
    int *seg_part = seg_end + kMaxSegments;
    int *seg_first = seg_part + kMaxSegments;
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

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
            ptx::mbar_init(&p_full[i], 4);      // one arrival per softmax warp
        }
        ptx::mbar_init(o_bar, 1);
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_base_slot, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;
    // TMEM columns: S buffer st at st*128, O accumulator of partition q at 256 + q*HD
    auto tS = [tmem](int st) { return tmem + (uint32_t)st * 128u; };
    auto tO = [tmem](int q) { return tmem + 256u + (uint32_t)q * (uint32_t)HD; };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmQ);
            ptx::tma_prefetch_desc(&tmK);
            ptx::tma_prefetch_desc(&tmV);
            const uint64_t pol_q = ptx::policy_evict_first();
            const uint64_t pol_kv = ptx::policy_evict_last();
            ptx::mbar_arrive_expect_tx(q_full, L::kQBytes);
            for (int b = 0; b < HD / 64; ++b)
                ptx::tma_load_3d(sQ + b * (kBlockM * 128), &tmQ, q_full, b * 64, head, q0, pol_q);
            TileCursor cur;
            cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
            int issued = -1;
            bool ok = true;
            for (int j = 0; j < n_tiles; ++j, cur.advance()) {
                const int st = j % NS;
                ok = ptx::mbar_wait_bounded(&kv_empty[st], ((j / NS) & 1) ^ 1, kWaitLimitNs, p.err_flag, abort_flag);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(&kv_full[st], 2 * L::kKVBytes);
                for (int b = 0; b < HD / 64; ++b) {
                    ptx::tma_load_3d(sK + st * L::kKVBytes + b * (kBlockN * 128), &tmK, &kv_full[st], b * 64, head,
                                     cur.row0, pol_kv);
                    ptx::tma_load_3d(sV + st * L::kKVBytes + b * (kBlockN * 128), &tmV, &kv_full[st], b * 64, head,
                                     cur.row0, pol_kv);
                }
                issued = j;
            }
            if (!ok) {
                // drain copies that may still be writing shared memory
                for (int j = issued - NS + 1 > 0 ? issued - NS + 1 : 0; j <= issued; ++j)
                    ptx::mbar_wait_bounded(&kv_full[j % NS], (j / NS) & 1, kWaitLimitNs, nullptr, nullptr);
                ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, nullptr, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = ptx::make_idesc_bf16(kBlockM, kBlockN, false, false);
            constexpr uint32_t idesc_pv = ptx::make_idesc_bf16(kBlockM, HD, false, true);
            const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aV = ptx::smem_u32(sV);
            bool ok = ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, p.err_flag, abort_flag);
            // S_j = Q K_j^T into S buffer j%2 (waits for K_j and V_j: they land together)
            auto issue_s = [&](int j) -> bool {
                const int sb = j & 1, ks = j % NS;
                if (!ptx::mbar_wait_bounded(&kv_full[ks], (j / NS) & 1, kWaitLimitNs, p.err_flag, abort_flag))
                    return false;
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t koff = (kk / 4) * (kBlockM * 128) + (kk % 4) * 32;
                    const uint64_t da = ptx::make_sdesc_sw128(aQ + koff, 16, 1024);
                    const uint64_t db = ptx::make_sdesc_sw128(aK + ks * L::kKVBytes + koff, 16, 1024);
                    ptx::umma_f16_ss(tS(sb), da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::umma_commit(&s_full[sb]);
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
                ok = ptx::mbar_wait_bounded(&p_full[sb], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                // O += P V with P (bf16) in the first 64 columns of S buffer sb: 16 keys = 8 columns per step
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint64_t db = ptx::make_sdesc_sw128(aV + vs * L::kKVBytes + kk * 2048, kBlockN * 128, 1024);
                    ptx::umma_f16_ts(dO, tS(sb) + kk * 8, db, idesc_pv, kk > 0 ? 1u : acc0);
                }
                ptx::umma_commit(o_bar);
                ptx::umma_commit(&kv_empty[vs]);
            }
            // all MMAs issued by this thread must finish before TMEM is released
            ptx::umma_commit(done_bar);
            ptx::mbar_wait_bounded(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp - kSoftmaxWarp0;          // TMEM lane quarter
        const int row = wq * 32 + lane;               // query row inside the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        float m_loc = -INFINITY, m_hist = -INFINITY;   // reference maxima (log2 units)
        float l_loc = 0.f, l_hist = 0.f;               // softmax denominators
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
            const int st = j & 1;
            const int valid = cur.valid();
            const int part = cur.part;
            ok = ptx::mbar_wait_bounded(&s_full[st], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            // all four 32-column loads in flight before one wait
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
            // row maximum: four independent chains of 3-input max
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
            const float mref = m_cur;
            // exponentials, eight independent partial sums, bf16 pairs for P
            float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[kBlockN / 2];
            const float neg_m = -mref;
#pragma unroll
            for (int c = 0; c < kBlockN; c += 2) {
                // one column in four goes to the FMA-pipe exponential, the rest to MUFU
                const float e0 = ptx::exp2_approx(fmaf(s[c], p.scale_log2, neg_m));
                const float x1 = fmaf(s[c + 1], p.scale_log2, neg_m);
                const float e1 = ((c / 2) % 2 == 1) ? ptx::exp2_poly(x1) : ptx::exp2_approx(x1);
                sum8[(c / 2) % 8] += e0 + e1;
                pk[c / 2] = pack_bf16x2(e0, e1);
            }
            const float rowsum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            l_cur = fmaf(l_cur, alpha, rowsum);
            if (part) { m_hist = m_cur; l_hist = l_cur; } else { m_loc = m_cur; l_loc = l_cur; }
            // P (row `row`: 128 bf16 packed in 64 columns) over the first half of this S buffer,
            // the A operand of the PV MMA
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
                ok = ptx::mbar_wait_bounded(o_bar, (j - 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
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
            if (lane == 0) ptx::mbar_arrive(&p_full[st]);
        }
        // ---------------------------------------------------------------- epilogue
        if (ok && n_tiles > 0) ok = ptx::mbar_wait_bounded(o_bar, (n_tiles - 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
        if (ok) {
            ptx::tc_fence_after();
            const int qrow = q0 + row;
            const bool active = qrow < p.n_q;
            constexpr float kLn2 = 0.69314718055994530942f;
            float L2[2];
            L2[0] = l_loc > 0.f ? m_loc + log2f(l_loc) : -INFINITY;
            L2[1] = l_hist > 0.f ? m_hist + log2f(l_hist) : -INFINITY;
            const float mx = fmaxf(L2[0], L2[1]);
            float w_loc = 0.f, w_hist = 0.f, lse_full = -INFINITY;
            if (mx != -INFINITY) {
                const float el = exp2f(L2[0] - mx), eh = exp2f(L2[1] - mx);
                w_loc = el / (el + eh);
                w_hist = eh / (el + eh);
                lse_full = (mx + log2f(el + eh)) * kLn2;
            }
            const float inv_l[2] = {l_loc > 0.f ? 1.f / l_loc : 0.f, l_hist > 0.f ? 1.f / l_hist : 0.f};
            const bool has[2] = {l_loc > 0.f, l_hist > 0.f};
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
                    const float al0 = has[0] ? __uint_as_float(rl[i]) * inv_l[0] : 0.f;
                    const float al1 = has[0] ? __uint_as_float(rl[i + 1]) * inv_l[0] : 0.f;
                    const float ah0 = has[1] ? __uint_as_float(rh[i]) * inv_l[1] : 0.f;
                    const float ah1 = has[1] ? __uint_as_float(rh[i + 1]) * inv_l[1] : 0.f;
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
                if (p.lse_loc) p.lse_loc[li] = L2[0] == -INFINITY ? -INFINITY : L2[0] * kLn2;
                if (p.lse_hist) p.lse_hist[li] = L2[1] == -INFINITY ? -INFINITY : L2[1] * kLn2;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows, heads, hd] bf16 tensor, box = 128 rows x 64 columns of one head, 128-byte swizzle.
bool make_rows_map(CUtensorMap *m, const void *ptr, int rows, int heads, int hd) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)heads * hd * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_hd(const AttnArgs &a, cudaStream_t s) {
    CUtensorMap mq, mk, mv;
    const void *kp = a.n_kv > 0 ? a.k : a.q;
    const void *vp = a.n_kv > 0 ? a.v : a.q;
    const int kv_rows = a.n_kv > 0 ? a.n_kv : a.n_q;
    if (!make_rows_map(&mq, a.q, a.n_q, a.heads, HD) || !make_rows_map(&mk, kp, kv_rows, a.heads, HD) ||
        !make_rows_map(&mv, vp, kv_rows, a.heads, HD))
        return cudaErrorInvalidValue;
    SplitParams p;
    p.o_full = a.o_full; p.lse_full = a.lse_full;
    p.o_loc = a.o_loc; p.lse_loc = a.lse_loc;
    p.o_hist = a.o_hist; p.lse_hist = a.lse_hist;
    p.a_ops = a.a_loc_ops; p.r_ops = a.r_ops;
    p.n_q = a.n_q; p.heads = a.heads;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.segs = a.segs;
    p.err_flag = a.err_flag;
    constexpr int smem = Smem<HD>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_split_sm100_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.n_q + kBlockM - 1) / kBlockM, a.heads);
    attn_split_sm100_kernel<HD><<<grid, kThreads, smem, s>>>(mq, mk, mv, p); note_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const AttnArgs &a, cudaStream_t s) {
    if (a.n_q == 0) return cudaSuccess;
    if (a.head_dim == 128) return launch_hd<128>(a, s);
    if (a.head_dim == 64) return launch_hd<64>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ispa
