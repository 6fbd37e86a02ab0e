// Split (decomposable) attention on the sm_100a tensor cores, bf16 operands, float32
// softmax and accumulation [ISPA §3.1 step 1 "Dual-Stream Warmup", §3.4 "Decomposable
// Attention"].
//
// One pass over the KV rows of one layer keeps two online-softmax states per query row:
// the local partition (sink frame + current chunk) and the history partition (all other
// rows). The epilogue merges them by their log-sum-exps into the full output, so the full
// and the local attention cost one attention pass. It also forms the statistics operands
// A_loc and R = A_full - A_loc = w_hist (A_hist - A_loc) in registers and stores them
// (bf16) for the statistics GEMM that follows on the same stream.
//
// The KV tiles are visited partition by partition (every local tile, then every history
// tile), so only one float32 accumulator O is live in tensor memory at a time. When the
// walk crosses from the local to the history partition, the softmax warps read the
// finished local accumulator, normalise it (A_loc, rounded to bf16 -- the precision every
// output of this kernel has) into shared memory, and the first history PV restarts O from
// zero. That frees the tensor memory for a third S buffer.
//
// CTA = one 128-row query tile of one head; 256 threads:
//   warp 0      TMA producer: Q once, then K tiles into a 3-deep ring
//   warp 1      TMEM allocation; issues every tcgen05.mma and commit
//   warp 2      TMA producer: V tiles into a 2-deep ring
// (the producer and MMA warps stay converged; one elected lane issues each instruction)
//   warps 4..7  softmax (thread i owns query row i = TMEM lane i), lazy rescale, epilogue
// TMEM (512 columns): three S buffers (3 x 128) and O (HD). P (bf16) is written over the
// first 64 columns of the S buffer it came from and feeds the PV MMA straight from tensor
// memory. Shared memory: Q, the K and V rings (TMA, 128-byte swizzle) and the A_loc spill.
//
// MMA order S_0, S_1, S_2, PV_0, S_3, PV_1, ...: two S tiles run ahead of the softmax, so
// the tensor pipe has work queued while a finished S travels to the softmax warps and its P
// travels back. tcgen05.mma operations of one thread execute in issue order, so S_{j+3}
// (which overwrites S buffer j%3, holding P_j) starts only after PV_j has consumed P_j, and
// the completion of S_j implies that of PV_{j-3}. PV_j commits to barrier o_bar[j%3]: with
// one barrier per buffer the phase a softmax warp waits for is never more than one phase
// away from the barrier's current one, so its parity waits are exact even though a warp
// waits on O only when it has to (a rescale, the partition switch, the epilogue).
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
constexpr int kNumS = 3;       // S/P buffers in tensor memory
constexpr int kKStages = 3;    // K ring depth
constexpr int kVStages = 2;    // V ring depth
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;          // log2 units: rescale when the max grows by > 2^8
// Column pairs (by index mod 8) whose exponentials run on the FMA pipe instead of MUFU: one
// pair in four (measured best on a 1.3B layer call among 0, 1/4, 3/8, 1/2 and 5/8).
constexpr unsigned kPolyPairs = 0x22;

template <int HD>
struct Smem {
    static constexpr int kQBytes = kBlockM * HD * 2;
    static constexpr int kKVBytes = kBlockN * HD * 2;    // one K or V tile
    static constexpr int kSpillBytes = kBlockM * HD * 2; // A_loc, bf16
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;
    static constexpr int kV = kK + kKStages * kKVBytes;
    static constexpr int kSpill = kV + kVStages * kKVBytes;
    static constexpr int kBar = kSpill + kSpillBytes;
    // q, k full/empty, v full/empty, s_full, p_full, o_bar, done
    static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 3 * kNumS + 1;
    static constexpr int kSeg = kBar + kNumBars * 8;      // segment table: 4 x kMaxSegments ints
    static constexpr int kMisc = kSeg + 4 * kMaxSegments * 4;
    static constexpr int kTotal = kMisc + 16;
    static constexpr int kAlloc = kTotal + 1024;          // slack for 1024-byte alignment
    static_assert(kAlloc <= 232448, "shared memory budget");
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
    SegmentList segs;   // local segments first, then history segments
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
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Byte offset of 16-byte chunk c of spill row r: chunks are XOR-swizzled by r % 8 so that a
// warp storing one chunk per row touches all 32 banks.
template <int HD>
__device__ __forceinline__ uint32_t spill_off(int r, int c) {
    return (uint32_t)r * (HD * 2) + (uint32_t)((c ^ (r & 7)) * 16);
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
attn_split_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const SplitParams p) {
    using L = Smem<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::kQ;
    uint8_t *sK = smem + L::kK;
    uint8_t *sV = smem + L::kV;
    uint8_t *sSpill = smem + L::kSpill;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = q_full + 1;            // [kKStages] K tile landed
    uint64_t *k_empty = k_full + kKStages;    // [kKStages] S of that tile done
    uint64_t *v_full = k_empty + kKStages;    // [kVStages] V tile landed
    uint64_t *v_empty = v_full + kVStages;    // [kVStages] PV of that tile done
    uint64_t *s_full = v_empty + kVStages;    // [kNumS] S buffer written by the MMA
    uint64_t *p_full = s_full + kNumS;        // [kNumS] P written (O rescaled / spilled) by the softmax
    uint64_t *o_bar = p_full + kNumS;         // [kNumS] PV of the tile in that buffer done
    uint64_t *done_bar = o_bar + kNumS;       //         every MMA of this CTA finished
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

    // The walk must see every local tile before the first history tile (one accumulator);
    // the host orders the segments that way. Anything else is refused before any barrier use.
    int n_tiles = 0;
    bool ordered = true;
    for (int s = 0; s < nseg; ++s) {
        n_tiles += (p.segs.seg[s].end - p.segs.seg[s].begin + kBlockN - 1) / kBlockN;
        if (s > 0 && p.segs.seg[s].part < p.segs.seg[s - 1].part) ordered = false;
    }
    if (!ordered) {
        if (threadIdx.x == 0) raise_device_error(p.err_flag, ISPA_ERR_UNSUPPORTED);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < nseg; ++s) {
            const Segment sg = p.segs.seg[s];
            seg_begin[s] = sg.begin;
            seg_end[s] = sg.end;
            seg_part[s] = sg.part;
            seg_first[s] = (s == 0 || p.segs.seg[s - 1].part != sg.part) ? 1 : 0;
        }
        ptx::mbar_init(q_full, 1);
        for (int i = 0; i < kKStages; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < kNumS; ++i) {
            ptx::mbar_init(&s_full[i], 1);
            ptx::mbar_init(&p_full[i], 4);      // one arrival per softmax warp
            ptx::mbar_init(&o_bar[i], 1);
        }
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
    // TMEM columns: S buffer b at b*128, the O accumulator at 384
    auto tS = [tmem](int b) { return tmem + (uint32_t)b * 128u; };
    const uint32_t tO = tmem + 384u;

    // Producer and MMA warps run their loops with all 32 lanes; one elected lane issues each
    // copy, MMA and commit (the *_warp helpers), so descriptors stay in uniform registers.
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer: Q, K
        const uint64_t pol_q = ptx::policy_evict_first();
        const uint64_t pol_kv = ptx::policy_evict_last();
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmQ);
            ptx::tma_prefetch_desc(&tmK);
        }
        ptx::mbar_arrive_expect_tx_warp(q_full, L::kQBytes);
#pragma unroll
        for (int b = 0; b < HD / 64; ++b) ptx::tma_load_3d_warp(sQ + b * (kBlockM * 128), &tmQ, q_full, b * 64, head, q0, pol_q);
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        int issued = -1;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j, cur.advance()) {
            const int st = j % kKStages;
            ok = ptx::mbar_wait_bounded(&k_empty[st], ((j / kKStages) & 1) ^ 1, kWaitLimitNs, p.err_flag, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ptx::mbar_arrive_expect_tx_warp(&k_full[st], L::kKVBytes);
#pragma unroll
            for (int b = 0; b < HD / 64; ++b)
                ptx::tma_load_3d_warp(sK + st * L::kKVBytes + b * (kBlockN * 128), &tmK, &k_full[st], b * 64, head,
                                      cur.row0, pol_kv);
            issued = j;
        }
        if (!ok) {
            // drain copies that may still be writing shared memory
            for (int j = issued - kKStages + 1 > 0 ? issued - kKStages + 1 : 0; j <= issued; ++j)
                ptx::mbar_wait_bounded(&k_full[j % kKStages], (j / kKStages) & 1, kWaitLimitNs, nullptr, nullptr);
            ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, nullptr, nullptr);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ TMA producer: V
        const uint64_t pol_kv = ptx::policy_evict_last();
        if (lane == 0) ptx::tma_prefetch_desc(&tmV);
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        int issued = -1;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j, cur.advance()) {
            const int st = j % kVStages;
            ok = ptx::mbar_wait_bounded(&v_empty[st], ((j / kVStages) & 1) ^ 1, kWaitLimitNs, p.err_flag, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ptx::mbar_arrive_expect_tx_warp(&v_full[st], L::kKVBytes);
#pragma unroll
            for (int b = 0; b < HD / 64; ++b)
                ptx::tma_load_3d_warp(sV + st * L::kKVBytes + b * (kBlockN * 128), &tmV, &v_full[st], b * 64, head,
                                      cur.row0, pol_kv);
            issued = j;
        }
        if (!ok) {
            for (int j = issued - kVStages + 1 > 0 ? issued - kVStages + 1 : 0; j <= issued; ++j)
                ptx::mbar_wait_bounded(&v_full[j % kVStages], (j / kVStages) & 1, kWaitLimitNs, nullptr, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_qk = ptx::make_idesc_bf16(kBlockM, kBlockN, false, false);
        constexpr uint32_t idesc_pv = ptx::make_idesc_bf16(kBlockM, HD, false, true);
        const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aV = ptx::smem_u32(sV);
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, p.err_flag, abort_flag));
        // S_j = Q K_j^T into S buffer j%3; frees K slot j%3 when done
        auto issue_s = [&](int j) -> bool {
            const int sb = j % kNumS, ks = j % kKStages;
            const bool w = ptx::mbar_wait_bounded(&k_full[ks], (j / kKStages) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (!__all_sync(0xffffffffu, w)) return false;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
                const uint32_t koff = (kk / 4) * (kBlockM * 128) + (kk % 4) * 32;
                const uint64_t da = ptx::make_sdesc_sw128(aQ + koff, 16, 1024);
                const uint64_t db = ptx::make_sdesc_sw128(aK + ks * L::kKVBytes + koff, 16, 1024);
                ptx::umma_f16_ss_warp(tS(sb), da, db, idesc_qk, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit_warp(&s_full[sb]);
            ptx::umma_commit_warp(&k_empty[ks]);
            return true;
        };
        if (ok && n_tiles > 0) ok = issue_s(0);
        if (ok && n_tiles > 1) ok = issue_s(1);
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
            if (j + 2 < n_tiles) {
                ok = issue_s(j + 2);
                if (!ok) break;
            }
            const int sb = j % kNumS, vs = j % kVStages;
            const uint32_t acc0 = cur.first_of_part() ? 0u : 1u;
            bool w = ptx::mbar_wait_bounded(&p_full[sb], (j / kNumS) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (w) w = ptx::mbar_wait_bounded(&v_full[vs], (j / kVStages) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            ptx::tc_fence_after();
            // O += P V with P (bf16) in the first 64 columns of S buffer sb: 16 keys = 8 columns per step
#pragma unroll
            for (int kk = 0; kk < kBlockN / 16; ++kk) {
                const uint64_t db = ptx::make_sdesc_sw128(aV + vs * L::kKVBytes + kk * 2048, kBlockN * 128, 1024);
                ptx::umma_f16_ts_warp(tO, tS(sb) + kk * 8, db, idesc_pv, kk > 0 ? 1u : acc0);
            }
            ptx::umma_commit_warp(&o_bar[sb]);
            ptx::umma_commit_warp(&v_empty[vs]);
        }
        // all MMAs issued by this warp must finish before TMEM is released
        ptx::umma_commit_warp(done_bar);
        ptx::mbar_wait_bounded(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp - kSoftmaxWarp0;          // TMEM lane quarter
        const int row = wq * 32 + lane;               // query row inside the tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;          // state of the partition being walked (log2 units)
        float m_loc = -INFINITY, l_loc = 0.f;          // the local partition's final state, once spilled
        int part_run = -1;
        bool spilled = false;
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, seg_first, nseg);
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
            const int sb = j % kNumS;
            const int valid = cur.valid();
            bool spill_now = false;
            if (cur.part != part_run) {
                // a new partition starts; the local one (if any tile of it ran) is spilled below
                spill_now = part_run == 0;
                if (spill_now) { m_loc = m_run; l_loc = l_run; }
                part_run = cur.part;
                m_run = -INFINITY;
                l_run = 0.f;
            }
            ok = ptx::mbar_wait_bounded(&s_full[sb], (j / kNumS) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            // all four 32-column loads in flight before one wait
            uint32_t sr[kBlockN];
#pragma unroll
            for (int c = 0; c < kBlockN / 32; ++c)
                ptx::tmem_ld32(tS(sb) + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            ptx::tmem_wait_ld();
            float *s = reinterpret_cast<float *>(sr);

            if (valid < kBlockN) {
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            // row maximum: eight independent chains of 3-input max (16 columns each)
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                mx8[u] = s[16 * u];
#pragma unroll
                for (int c = 1; c < 15; c += 2) mx8[u] = ptx::max3(mx8[u], s[16 * u + c], s[16 * u + c + 1]);
                mx8[u] = fmaxf(mx8[u], s[16 * u + 15]);
            }
            float mx = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]), ptx::max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
            mx *= p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_run + kRescaleThreshold || m_run == -INFINITY) {
                if (m_run != -INFINITY) {
                    alpha = exp2f(m_run - mx);
                    rescale = true;
                }
                m_run = mx;
            }
            // Exponentials by column pairs in packed float32 arithmetic: x = s * scale - m for
            // both columns in one instruction, the pair's 2^x either on MUFU (two ex2) or on
            // the FMA pipe (exp2_poly2) as kPolyPairs selects, four packed
            // partial sums, and the bf16 pair for P. MUFU and FMA-pipe pairs alternate so that
            // one warp keeps both units busy.
            uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
            uint32_t pk[kBlockN / 2];
            const uint64_t sc2 = ptx::f2_pack(p.scale_log2, p.scale_log2);
            const uint64_t nm2 = ptx::f2_pack(-m_run, -m_run);
#pragma unroll
            for (int q = 0; q < kBlockN / 2; ++q) {
                const uint64_t x2 = ptx::f2_fma(ptx::f2_pack(s[2 * q], s[2 * q + 1]), sc2, nm2);
                uint64_t e2;
                if ((kPolyPairs >> (q % 8)) & 1)
                    e2 = ptx::exp2_poly2(x2);
                else
                    e2 = ptx::f2_pack(ptx::exp2_approx(ptx::f2_lo(x2)), ptx::exp2_approx(ptx::f2_hi(x2)));
                acc2[q % 4] = ptx::f2_add(acc2[q % 4], e2);
                pk[q] = pack_bf16x2(ptx::f2_lo(e2), ptx::f2_hi(e2));
            }
            const uint64_t a01 = ptx::f2_add(acc2[0], acc2[1]), a23 = ptx::f2_add(acc2[2], acc2[3]);
            const uint64_t a4 = ptx::f2_add(a01, a23);
            const float rowsum = ptx::f2_lo(a4) + ptx::f2_hi(a4);
            l_run = fmaf(l_run, alpha, rowsum);
            // P (row `row`: 128 bf16 packed in 64 columns) over the first half of this S buffer,
            // the A operand of the PV MMA
            ptx::tmem_st32(tS(sb) + lane_off, &pk[0]);
            ptx::tmem_st32(tS(sb) + lane_off + 32, &pk[32]);
            ptx::tmem_wait_st();
            // O is touched only once PV_{j-1} is complete; without a rescale or a spill nothing
            // here waits for it.
            const bool rescale_warp = __any_sync(0xffffffffu, rescale);
            if ((rescale_warp || spill_now) && j >= 1) {
                const int pj = j - 1;
                ok = ptx::mbar_wait_bounded(&o_bar[pj % kNumS], (pj / kNumS) & 1, kWaitLimitNs, p.err_flag,
                                            abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
            }
            if (spill_now) {
                // A_loc = O / l_loc (bf16) into this row of the spill; the next PV overwrites O
                const float inv = l_loc > 0.f ? 1.f / l_loc : 0.f;
#pragma unroll 1
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t r[32];
                    ptx::tmem_ld32(tO + lane_off + c * 32, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 u;
                        u.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
                        u.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
                        u.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
                        u.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
                        *reinterpret_cast<uint4 *>(sSpill + spill_off<HD>(row, c * 4 + v)) = u;
                    }
                }
                spilled = true;
            } else if (rescale_warp) {
#pragma unroll
                for (int c = 0; c < HD / 16; ++c) {
                    uint32_t r[16];
                    ptx::tmem_ld16(tO + lane_off + c * 16, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    ptx::tmem_st16(tO + lane_off + c * 16, r);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&p_full[sb]);
        }
        // ---------------------------------------------------------------- epilogue
        if (ok && n_tiles > 0) {
            const int pj = n_tiles - 1;
            ok = ptx::mbar_wait_bounded(&o_bar[pj % kNumS], (pj / kNumS) & 1, kWaitLimitNs, p.err_flag, abort_flag);
        }
        if (ok) {
            ptx::tc_fence_after();
            // final states: O holds the partition walked last
            float m_hist = -INFINITY, l_hist = 0.f;
            if (part_run == 1) {
                m_hist = m_run;
                l_hist = l_run;
            } else if (part_run == 0) {
                m_loc = m_run;
                l_loc = l_run;
            }
            const int qrow = q0 + row;
            const bool active = qrow < p.n_q;
            constexpr float kLn2 = 0.69314718055994530942f;
            const float L2l = l_loc > 0.f ? m_loc + log2f(l_loc) : -INFINITY;
            const float L2h = l_hist > 0.f ? m_hist + log2f(l_hist) : -INFINITY;
            const float mxl = fmaxf(L2l, L2h);
            float w_loc = 0.f, w_hist = 0.f, lse_full = -INFINITY;
            if (mxl != -INFINITY) {
                const float el = exp2f(L2l - mxl), eh = exp2f(L2h - mxl);
                w_loc = el / (el + eh);
                w_hist = eh / (el + eh);
                lse_full = (mxl + log2f(el + eh)) * kLn2;
            }
            const bool has_run = l_run > 0.f;   // false when no tile ran (O never written)
            const float inv_run = has_run ? 1.f / l_run : 0.f;
            const bool o_is_hist = part_run == 1;
            const size_t D = (size_t)p.heads * HD;
            const size_t obase = ((size_t)qrow * p.heads + head) * HD;
            const size_t sbase = (size_t)qrow * D + (size_t)head * HD;
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t ro[32];
                ptx::tmem_ld32(tO + lane_off + c * 32, ro);
                ptx::tmem_wait_ld();
                if (!active) continue;
                // this row's 32 A_loc values of the chunk, from the spill (bf16 pairs)
                uint32_t sl[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 u = spilled ? *reinterpret_cast<const uint4 *>(sSpill + spill_off<HD>(row, c * 4 + v))
                                      : make_uint4(0u, 0u, 0u, 0u);
                    sl[4 * v] = u.x; sl[4 * v + 1] = u.y; sl[4 * v + 2] = u.z; sl[4 * v + 3] = u.w;
                }
                uint32_t of[16], ol[16], oh[16], orr[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float o0 = has_run ? __uint_as_float(ro[i]) * inv_run : 0.f;
                    const float o1 = has_run ? __uint_as_float(ro[i + 1]) * inv_run : 0.f;
                    const float al0 = o_is_hist ? bf16_lo(sl[i / 2]) : o0;
                    const float al1 = o_is_hist ? bf16_hi(sl[i / 2]) : o1;
                    const float ah0 = o_is_hist ? o0 : 0.f;
                    const float ah1 = o_is_hist ? o1 : 0.f;
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
    // local segments first (stable), as the kernel's single accumulator requires
    p.segs.count = 0;
    for (int part = 0; part < 2; ++part)
        for (int i = 0; i < a.segs.count; ++i)
            if (a.segs.seg[i].part == part) p.segs.seg[p.segs.count++] = a.segs.seg[i];
    if (p.segs.count != a.segs.count) return cudaErrorInvalidValue;
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
