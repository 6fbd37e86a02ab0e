// Split (decomposable) attention for head_dim 128 with two softmax groups per CTA
// [ISPA §3.1 step 1 "Dual-Stream Warmup", §3.4 "Decomposable Attention"].
//
// Same result as the single-group kernel (per query row: the local and the history
// partition's softmax states, merged by log-sum-exp; the statistics operands A_loc and R),
// organised so that two independent softmax warps share each SM sub-partition. The KV tiles
// alternate between two groups of four softmax warps: group g takes tiles j = g, g + 2, ...
// and keeps its own S buffer, O accumulator and running (m, l) per partition in tensor
// memory and registers. While one group computes the exponentials of its tile, the tensor
// pipe runs the other group's PV and next S, and the two groups' MUFU and FMA work interleave
// on the sub-partitions. At the end the groups' partial states are merged by log-sum-exp,
// like the partitions.
//
// CTA = one 128-row query tile of one head; 384 threads in three warpgroups:
//   warp 0      TMA producer: Q, then K tiles (2-deep ring)
//   warp 1      TMEM allocation; issues every tcgen05.mma and commit
//   warp 2      TMA producer: V tiles (2-deep ring)
//   warp 3      idle
//   warps 4..7  softmax group 0, warps 8..11 softmax group 1 (TMEM lane quarter = warp % 4)
// The first warpgroup gives registers back (setmaxnreg) so that each softmax thread can hold
// a whole 128-column S row; the host checks before the launch that the split fits the
// registers the kernel is launched with.
// TMEM (512 columns): S_0, S_1 (one 128-column buffer per group), O_0, O_1 (HD each). P (bf16)
// goes over the first 64 columns of the group's S buffer.
// Shared memory: Q, the K and V rings, and the local state (fp32, 64 KB, with its per-row m
// and l) that the groups hand over when they reach the history.
//
// MMA order S_0, S_1, PV_0, S_2, PV_1, S_3, ...: S_{j+2} (group j % 2) is issued right after
// PV_j, so the completion of S_j implies that of PV_{j-2} -- the group's previous PV: a group
// may rescale or read its accumulator as soon as its S tile is ready. Both groups walk the
// local tiles first. The group that meets the first history tile writes its local state,
// normalised, to the fp32 buffer; the other one, on meeting its own first history tile, waits
// for that and merges its local state into the buffer in fp32, so that A_loc is rounded to
// bf16 only once, on output. The epilogue waits for every MMA, exchanges the per-row states
// of the two groups through shared memory (the Q area, no longer read), and each group merges
// and stores half of the output columns.
//
// 8-bit variant (kI8) [ISPA §3.4 builds on 8-bit attention kernels, SageAttention]: Q and K
// arrive as int8 with a scale per (token, head) for Q and per (128-row block of a partition
// segment, head) for K; S = Q8 K8^T runs as tcgen05 kind::i8 (exact int32 accumulation, half
// the bytes and twice the rate of the bf16 MMA); V, P, PV and everything after stay as in the
// bf16 path. The softmax reads each int32 score as the float bits of 1.5 * 2^23 + s (one
// integer add; exact while |s| < 2^22, and |s| <= 128 * 127 * 127) and folds the offset and
// the per-row, per-tile scale s_q s_k into the FMA that forms the exponent.
//
// Every mbarrier wait is bounded; on timeout the CTA records ISPA_ERR_TIMEOUT in the device
// flag and every role leaves its loop.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ispa {
namespace {

constexpr int HD = 128;
constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kRegsLow = 56;    // producer / MMA warpgroup after setmaxnreg.dec
constexpr int kRegsHigh = 216;  // softmax warpgroups after setmaxnreg.inc
// registers one CTA needs after the split (checked against the launch's allocation)
constexpr int kRegsNeeded = 128 * kRegsLow + 256 * kRegsHigh;
constexpr int kStages = 2;     // K ring and V ring depth
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;
constexpr unsigned kPolyPairs = 0x22;   // column pairs (index mod 8) on the FMA-pipe exponential

// Shared-memory layout; Q and K tiles hold 1-byte (kI8) or 2-byte elements.
template <bool kI8>
struct Layout {
    static constexpr int kQKElem = kI8 ? 1 : 2;
    static constexpr int kQBytes = kBlockM * HD * kQKElem;
    static constexpr int kKBytes = kBlockN * HD * kQKElem;
    static constexpr int kVBytes = kBlockN * HD * 2;
    static constexpr int kBoxes = HD * kQKElem / 128;     // 128-byte-wide TMA boxes per Q/K row
    static constexpr int kSSteps = HD * kQKElem / 32;     // S MMAs per tile: 32 bytes of K each
    static constexpr int kSpillBytes = kBlockM * HD * 4;   // fp32 local state
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKBytes;
    static constexpr int kOffSpill = kOffV + kStages * kVBytes;
    static constexpr int kOffSpillML = kOffSpill + kSpillBytes;   // float m[128], l[128]
    static constexpr int kOffBar = kOffSpillML + 2 * kBlockM * 4;
    // q, k full/empty, v full/empty, s_full[2], p_full[2], spill, done
    static constexpr int kNumBars = 1 + 4 * kStages + 2 * 2 + 1 + 1;
    static constexpr int kOffSeg = kOffBar + kNumBars * 8;
    static constexpr int kOffMisc = kOffSeg + 4 * kMaxSegments * 4;
    static constexpr int kSmem = kOffMisc + 16 + 1024;   // + slack for 1024-byte alignment
};
static_assert(Layout<false>::kSmem <= 232448 && Layout<true>::kSmem <= 232448, "shared memory budget");

struct Split2gParams {
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
    SegmentList segs;   // local segments first, then history segments
    int *err_flag;
    // 8-bit variant: Q scales [n_q][heads], K scales [heads][n_blocks], and for each segment
    // (in the order above) the row-order index of its first K block
    const float *q_scale, *k_scale;
    int n_blocks;
    int seg_block0[kMaxSegments];
};

struct TileCursor {
    const int *sb, *se, *sp;
    int nseg, si, row0, end, part;
    __device__ __forceinline__ void init(const int *b, const int *e, const int *pt, int n) {
        sb = b; se = e; sp = pt; nseg = n; si = 0;
        if (n > 0) load();
    }
    __device__ __forceinline__ void load() { row0 = sb[si]; end = se[si]; part = sp[si]; }
    __device__ __forceinline__ void advance() {
        row0 += kBlockN;
        if (row0 >= end && ++si < nseg) load();
    }
    __device__ __forceinline__ int valid() const { return min(kBlockN, end - row0); }
    __device__ __forceinline__ int block(const int *blk0) const { return blk0[si] + (row0 - sb[si]) / kBlockN; }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Instruction descriptor, kind::i8: D s32, A and B signed 8-bit, both K-major.
__host__ __device__ constexpr uint32_t make_idesc_s8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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

__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow)); }
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh)); }

// barrier `id` over `nthreads` threads that also ANDs a flag across them
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Byte offset of 16-byte chunk c (4 floats, 0..31) of row r of the fp32 local state (chunks
// XOR-swizzled by r % 8: a warp storing one chunk per row touches all 32 banks).
__device__ __forceinline__ uint32_t spill_off(int r, int c) {
    return (uint32_t)r * (HD * 4) + (uint32_t)((c ^ (r & 7)) * 16);
}

template <bool kI8>
__global__ void __launch_bounds__(kThreads, 1)
attn_split_2g_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Split2gParams p) {
    using L = Layout<kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::kOffQ;
    uint8_t *sK = smem + L::kOffK;
    uint8_t *sV = smem + L::kOffV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *q_full = bars;
    uint64_t *k_full = q_full + 1;         // [kStages]
    uint64_t *k_empty = k_full + kStages;  // [kStages]
    uint64_t *v_full = k_empty + kStages;  // [kStages]
    uint64_t *v_empty = v_full + kStages;  // [kStages]
    uint64_t *s_full = v_empty + kStages;  // [2] per group
    uint64_t *p_full = s_full + 2;         // [2] per group (4 warps each)
    uint64_t *spill_bar = p_full + 2;      // the first group's local state is in the buffer
    uint64_t *done_bar = spill_bar + 1;
    int *seg_begin = reinterpret_cast<int *>(smem + L::kOffSeg);
    int *seg_end = seg_begin + kMaxSegments;
    int *seg_part = seg_end + kMaxSegments;
    int *seg_blk0 = seg_part + kMaxSegments;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int q0 = blockIdx.x * kBlockM;
    const int head = blockIdx.y;
    const int nseg = p.segs.count;
    int n_tiles = 0, n_local = 0;
    bool ordered = true;
    for (int s = 0; s < nseg; ++s) {
        const int t = (p.segs.seg[s].end - p.segs.seg[s].begin + kBlockN - 1) / kBlockN;
        n_tiles += t;
        if (p.segs.seg[s].part == 0) n_local += t;
        if (s > 0 && p.segs.seg[s].part < p.segs.seg[s - 1].part) ordered = false;
    }
    if (!ordered) {
        if (threadIdx.x == 0) raise_device_error(p.err_flag, ISPA_ERR_UNSUPPORTED);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < nseg; ++s) {
            seg_begin[s] = p.segs.seg[s].begin;
            seg_end[s] = p.segs.seg[s].end;
            seg_part[s] = p.segs.seg[s].part;
            seg_blk0[s] = p.seg_block0[s];
        }
        ptx::mbar_init(q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&k_empty[i], 1);
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&v_empty[i], 1);
        }
        for (int g = 0; g < 2; ++g) {
            ptx::mbar_init(&s_full[g], 1);
            ptx::mbar_init(&p_full[g], 4);
        }
        ptx::mbar_init(spill_bar, 4);
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto tS = [tmem](int g) { return tmem + (uint32_t)g * 128u; };
    auto tO = [tmem](int g) { return tmem + 256u + (uint32_t)g * 128u; };

    // Each role changes its register allocation at its own start (every warp of a warpgroup
    // takes the same setmaxnreg), so that the compiler sees one limit per role.
    if (warp == 0 || warp == 2) {
        regs_dec();
        // ------------------------------------------------------------ TMA producers
        // warp 0: Q, then K; warp 2: V. All lanes run the loop, one elected lane issues.
        const bool is_k = warp == 0;
        const CUtensorMap *tm = is_k ? &tmK : &tmV;
        // a K tile is kBoxes boxes of 128 bytes x 128 rows, a V tile two (bf16)
        const int tile_bytes = is_k ? L::kKBytes : L::kVBytes;
        const int boxes = is_k ? L::kBoxes : 2;
        const int box_cols = is_k ? 128 / L::kQKElem : 64;
        uint8_t *ring = is_k ? sK : sV;
        uint64_t *full = is_k ? k_full : v_full;
        uint64_t *empty = is_k ? k_empty : v_empty;
        const uint64_t pol_kv = ptx::policy_evict_last();
        if (lane == 0) ptx::tma_prefetch_desc(tm);
        if (is_k) {
            if (lane == 0) ptx::tma_prefetch_desc(&tmQ);
            ptx::mbar_arrive_expect_tx_warp(q_full, L::kQBytes);
#pragma unroll
            for (int b = 0; b < L::kBoxes; ++b)
                ptx::tma_load_3d_warp(sQ + b * (kBlockM * 128), &tmQ, q_full, b * (128 / L::kQKElem), head, q0,
                                      ptx::policy_evict_first());
        }
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, nseg);
        int issued = -1;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j, cur.advance()) {
            const int st = j % kStages;
            ok = ptx::mbar_wait_bounded(&empty[st], ((j / kStages) & 1) ^ 1, kWaitLimitNs, p.err_flag, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ptx::mbar_arrive_expect_tx_warp(&full[st], tile_bytes);
            for (int b = 0; b < boxes; ++b)
                ptx::tma_load_3d_warp(ring + st * tile_bytes + b * (kBlockN * 128), tm, &full[st], b * box_cols, head,
                                      cur.row0, pol_kv);
            issued = j;
        }
        if (!ok) {
            // drain copies that may still be writing shared memory
            for (int j = issued - kStages + 1 > 0 ? issued - kStages + 1 : 0; j <= issued; ++j)
                ptx::mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs, nullptr, nullptr);
            if (is_k) ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, nullptr, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (converged)
        regs_dec();
        constexpr uint32_t idesc_qk =
            kI8 ? make_idesc_s8(kBlockM, kBlockN) : ptx::make_idesc_bf16(kBlockM, kBlockN, false, false);
        constexpr uint32_t idesc_pv = ptx::make_idesc_bf16(kBlockM, HD, false, true);
        const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aV = ptx::smem_u32(sV);
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(q_full, 0, kWaitLimitNs, p.err_flag, abort_flag));
        auto issue_s = [&](int j) -> bool {
            const int g = j & 1, ks = j % kStages;
            const bool w = ptx::mbar_wait_bounded(&k_full[ks], (j / kStages) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (!__all_sync(0xffffffffu, w)) return false;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < L::kSSteps; ++kk) {
                const uint32_t koff = (kk / 4) * (kBlockM * 128) + (kk % 4) * 32;
                const uint64_t da = ptx::make_sdesc_sw128(aQ + koff, 16, 1024);
                const uint64_t db = ptx::make_sdesc_sw128(aK + ks * L::kKBytes + koff, 16, 1024);
                if constexpr (kI8)
                    umma_s8_ss_warp(tS(g), da, db, idesc_qk, kk > 0 ? 1u : 0u);
                else
                    ptx::umma_f16_ss_warp(tS(g), da, db, idesc_qk, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit_warp(&s_full[g]);
            ptx::umma_commit_warp(&k_empty[ks]);
            return true;
        };
        if (ok && n_tiles > 0) ok = issue_s(0);
        if (ok && n_tiles > 1) ok = issue_s(1);
        int part_last[2] = {-1, -1};
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, nseg);
        for (int j = 0; j < n_tiles && ok; ++j, cur.advance()) {
            const int g = j & 1, vs = j % kStages;
            const uint32_t acc0 = part_last[g] == cur.part ? 1u : 0u;   // the group's first tile of this partition
            part_last[g] = cur.part;
            bool w = ptx::mbar_wait_bounded(&p_full[g], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            if (w) w = ptx::mbar_wait_bounded(&v_full[vs], (j / kStages) & 1, kWaitLimitNs, p.err_flag, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBlockN / 16; ++kk)
                ptx::umma_f16_ts_warp(tO(g), tS(g) + kk * 8,
                                      ptx::make_sdesc_sw128(aV + vs * L::kVBytes + kk * 2048, kBlockN * 128, 1024),
                                      idesc_pv, kk > 0 ? 1u : acc0);
            ptx::umma_commit_warp(&v_empty[vs]);
            if (j + 2 < n_tiles) ok = issue_s(j + 2);
        }
        ptx::umma_commit_warp(done_bar);
        ptx::mbar_wait_bounded(done_bar, 0, kWaitLimitNs, p.err_flag, nullptr);
    } else if (warp == 3) {
        regs_dec();
    } else {
        regs_inc();
        // ------------------------------------------------------------ softmax + epilogue
        const int g = (warp - kSoftmaxWarp0) / 4;    // group
        const int wq = warp % 4;                     // TMEM lane quarter
        const int row = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        uint8_t *spill = smem + L::kOffSpill;
        float *spill_m = reinterpret_cast<float *>(smem + L::kOffSpillML);
        float *spill_l = spill_m + kBlockM;
        // the group of the first history tile hands its local state over first
        const int first_group = n_local & 1;
        const bool has_history = n_local < n_tiles;
        // exponent factor of a score (log2 units): the softmax scale, times s_q s_k for int8
        constexpr float kOff = kI8 ? 12582912.0f : 0.0f;   // 1.5 * 2^23: an int32 score's float offset
        float rsq = p.scale_log2;
        if constexpr (kI8)
            if (q0 + row < p.n_q) rsq *= p.q_scale[(size_t)(q0 + row) * p.heads + head];
        float m_run = -INFINITY, l_run = 0.f;    // this group's partition being walked
        int part_run = -1;
        TileCursor cur;
        cur.init(seg_begin, seg_end, seg_part, nseg);
        if (g == 1 && n_tiles > 0) cur.advance();
        bool ok = true;
        for (int j = g; j < n_tiles && ok; j += 2, cur.advance(), cur.advance()) {
            const int valid = cur.valid();
            float rs = rsq;
            // a zero scale comes only with all-zero scores (an all-zero Q row or K block): any
            // positive factor gives them the same exponent, and keeps -inf * rs = -inf on the
            // masked columns of a ragged tile (0 * -inf would be NaN)
            if constexpr (kI8) rs = fmaxf(rs * p.k_scale[(size_t)head * p.n_blocks + cur.block(seg_blk0)], 1.17549435e-38f);
            bool to_history = false, had_local = false;
            float m_prev = -INFINITY, l_prev = 0.f;
            if (cur.part != part_run) {
                to_history = cur.part == 1;
                had_local = part_run == 0;
                m_prev = m_run;
                l_prev = l_run;
                part_run = cur.part;
                m_run = -INFINITY;
                l_run = 0.f;
            }
            ok = __all_sync(0xffffffffu,
                            ptx::mbar_wait_bounded(&s_full[g], (j >> 1) & 1, kWaitLimitNs, p.err_flag, abort_flag));
            if (!ok) break;
            ptx::tc_fence_after();
            uint32_t sr[kBlockN];
#pragma unroll
            for (int c = 0; c < kBlockN / 32; ++c)
                ptx::tmem_ld32(tS(g) + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            ptx::tmem_wait_ld();
            if constexpr (kI8) {
#pragma unroll
                for (int c = 0; c < kBlockN; ++c) sr[c] += 0x4B400000u;   // float bits of 1.5 * 2^23 + score
            }
            float *s = reinterpret_cast<float *>(sr);
            if (valid < kBlockN) {
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                mx8[u] = s[16 * u];
#pragma unroll
                for (int c = 1; c < 15; c += 2) mx8[u] = ptx::max3(mx8[u], s[16 * u + c], s[16 * u + c + 1]);
                mx8[u] = fmaxf(mx8[u], s[16 * u + 15]);
            }
            const float mxr = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]), ptx::max3(mx8[3], mx8[4], mx8[5]),
                                        fmaxf(mx8[6], mx8[7]));
            const float mx = (kI8 ? mxr - kOff : mxr) * rs;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_run + kRescaleThreshold || m_run == -INFINITY) {
                if (m_run != -INFINITY) {
                    alpha = exp2f(m_run - mx);
                    rescale = true;
                }
                m_run = mx;
            }
            uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
            uint32_t pk[kBlockN / 2];
            // x = (s - kOff) rs - m as one FMA: s rs - (kOff rs + m)
            const float nm = kI8 ? -fmaf(kOff, rs, m_run) : -m_run;
            const uint64_t sc2 = ptx::f2_pack(rs, rs);
            const uint64_t nm2 = ptx::f2_pack(nm, nm);
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
            const uint64_t a4 = ptx::f2_add(ptx::f2_add(acc2[0], acc2[1]), ptx::f2_add(acc2[2], acc2[3]));
            l_run = fmaf(l_run, alpha, ptx::f2_lo(a4) + ptx::f2_hi(a4));
            ptx::tmem_st32(tS(g) + lane_off, &pk[0]);
            ptx::tmem_st32(tS(g) + lane_off + 32, &pk[32]);
            ptx::tmem_wait_st();
            // the group's previous PV (PV_{j-2}) completed before S_j did: O_g may be read now
            if (to_history && g == first_group) {
                // hand the local state over: O_g / l, with (m, l); nothing if the group had no local tile
                if (had_local) {
                    const float inv = l_prev > 0.f ? 1.f / l_prev : 0.f;
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        ptx::tmem_ld32(tO(g) + lane_off + c * 32, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            *reinterpret_cast<float4 *>(spill + spill_off(row, c * 8 + v)) =
                                make_float4(__uint_as_float(r[4 * v]) * inv, __uint_as_float(r[4 * v + 1]) * inv,
                                            __uint_as_float(r[4 * v + 2]) * inv, __uint_as_float(r[4 * v + 3]) * inv);
                    }
                }
                spill_m[row] = m_prev;
                spill_l[row] = l_prev;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(spill_bar);
            } else if (to_history && had_local) {
                // merge this group's local state into the buffer, in fp32
                ok = __all_sync(0xffffffffu,
                                ptx::mbar_wait_bounded(spill_bar, 0, kWaitLimitNs, p.err_flag, abort_flag));
                if (!ok) break;
                const float ms = spill_m[row], ls = spill_l[row];
                const float Ls = ls > 0.f ? ms + log2f(ls) : -INFINITY;
                const float Lb = l_prev > 0.f ? m_prev + log2f(l_prev) : -INFINITY;
                const float M = fmaxf(Ls, Lb);
                float cs = 0.f, cb = 0.f, E = 0.f;
                if (M != -INFINITY) {
                    const float es = ls > 0.f ? exp2f(Ls - M) : 0.f;
                    const float eb = l_prev > 0.f ? exp2f(Lb - M) : 0.f;
                    E = es + eb;
                    cs = es / E;
                    cb = l_prev > 0.f ? eb / (E * l_prev) : 0.f;
                }
                const bool use_s = cs > 0.f, use_b = cb > 0.f;
#pragma unroll 1
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t r[32];
                    ptx::tmem_ld32(tO(g) + lane_off + c * 32, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        float4 *dst = reinterpret_cast<float4 *>(spill + spill_off(row, c * 8 + v));
                        const float4 a = use_s ? *dst : make_float4(0.f, 0.f, 0.f, 0.f);
                        float4 o;
                        // selects, not products with zero: an unused buffer row may hold anything
                        o.x = (use_s ? a.x * cs : 0.f) + (use_b ? __uint_as_float(r[4 * v]) * cb : 0.f);
                        o.y = (use_s ? a.y * cs : 0.f) + (use_b ? __uint_as_float(r[4 * v + 1]) * cb : 0.f);
                        o.z = (use_s ? a.z * cs : 0.f) + (use_b ? __uint_as_float(r[4 * v + 2]) * cb : 0.f);
                        o.w = (use_s ? a.w * cs : 0.f) + (use_b ? __uint_as_float(r[4 * v + 3]) * cb : 0.f);
                        *dst = o;
                    }
                }
                spill_m[row] = M;
                spill_l[row] = E;
            } else if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int c = 0; c < HD / 16; ++c) {
                    uint32_t r[16];
                    ptx::tmem_ld16(tO(g) + lane_off + c * 16, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    ptx::tmem_st16(tO(g) + lane_off + c * 16, r);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&p_full[g]);
        }
        // ---------------------------------------------------------------- epilogue
        // every MMA of the CTA done (both groups' last PV; Q no longer read)
        ok = ok && ptx::mbar_wait_bounded(done_bar, 0, kWaitLimitNs, p.err_flag, abort_flag);
        // exchange (m, l, partition) of the last partition walked with the other group's warp of
        // the same lane quarter, through the Q area
        float *xq = reinterpret_cast<float *>(sQ);   // [2 groups][3][128 rows]
        if (ok) {
            xq[(g * 3 + 0) * kBlockM + row] = m_run;
            xq[(g * 3 + 1) * kBlockM + row] = l_run;
            xq[(g * 3 + 2) * kBlockM + row] = __int_as_float(part_run);
        }
        ok = named_bar_and(1, 256, ok);
        if (ok) {
            ptx::tc_fence_after();
            const float m0 = xq[0 * kBlockM + row], l0 = xq[1 * kBlockM + row];
            const int p0 = __float_as_int(xq[2 * kBlockM + row]);
            const float m1 = xq[3 * kBlockM + row], l1 = xq[4 * kBlockM + row];
            const int p1 = __float_as_int(xq[5 * kBlockM + row]);
            // local = the handed-over state (if any group reached the history) and every group
            // still in the local partition; history = every group in the history
            const float ms = has_history ? spill_m[row] : -INFINITY;
            const float ls = has_history ? spill_l[row] : 0.f;
            const float Ls = ls > 0.f ? ms + log2f(ls) : -INFINITY;
            const float L0 = l0 > 0.f ? m0 + log2f(l0) : -INFINITY;
            const float L1 = l1 > 0.f ? m1 + log2f(l1) : -INFINITY;
            const float L0l = p0 == 0 ? L0 : -INFINITY, L0h = p0 == 1 ? L0 : -INFINITY;
            const float L1l = p1 == 0 ? L1 : -INFINITY, L1h = p1 == 1 ? L1 : -INFINITY;
            const float Ml = ptx::max3(Ls, L0l, L1l), Mh = fmaxf(L0h, L1h);
            float L2l = -INFINITY, L2h = -INFINITY;
            float cs = 0.f, c0 = 0.f, c1 = 0.f;   // weights of the buffer, O_0, O_1 in their partition
            if (Ml != -INFINITY) {
                const float es = exp2f(Ls - Ml), e0 = exp2f(L0l - Ml), e1 = exp2f(L1l - Ml);
                const float El = es + e0 + e1;
                L2l = Ml + log2f(El);
                cs = es / El;
                if (p0 == 0) c0 = e0 / (El * l0);
                if (p1 == 0) c1 = e1 / (El * l1);
            }
            if (Mh != -INFINITY) {
                const float e0 = exp2f(L0h - Mh), e1 = exp2f(L1h - Mh);
                const float Eh = e0 + e1;
                L2h = Mh + log2f(Eh);
                if (p0 == 1) c0 = e0 / (Eh * l0);
                if (p1 == 1) c1 = e1 / (Eh * l1);
            }
            constexpr float kLn2 = 0.69314718055994530942f;
            const float mxl = fmaxf(L2l, L2h);
            float w_loc = 0.f, w_hist = 0.f, lse_full = -INFINITY;
            if (mxl != -INFINITY) {
                const float el = exp2f(L2l - mxl), eh = exp2f(L2h - mxl);
                w_loc = el / (el + eh);
                w_hist = eh / (el + eh);
                lse_full = (mxl + log2f(el + eh)) * kLn2;
            }
            const bool use_s = cs > 0.f;
            const bool u0l = p0 == 0 && c0 > 0.f, u0h = p0 == 1 && c0 > 0.f;
            const bool u1l = p1 == 0 && c1 > 0.f, u1h = p1 == 1 && c1 > 0.f;
            const int qrow = q0 + row;
            const bool active = qrow < p.n_q;
            const size_t D = (size_t)p.heads * HD;
            const size_t obase = ((size_t)qrow * p.heads + head) * HD;
            const size_t sbase = (size_t)qrow * D + (size_t)head * HD;
#pragma unroll 1
            for (int c = 2 * g; c < 2 * g + 2; ++c) {   // this group's 64 output columns
                uint32_t r0[32], r1[32];
                ptx::tmem_ld32(tO(0) + lane_off + c * 32, r0);
                ptx::tmem_ld32(tO(1) + lane_off + c * 32, r1);
                ptx::tmem_wait_ld();
                if (!active) continue;
                uint32_t of[16], ol[16], oh[16], orr[16];
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float4 sv = use_s ? *reinterpret_cast<const float4 *>(spill + spill_off(row, c * 8 + v))
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float svv[4] = {sv.x, sv.y, sv.z, sv.w};
                    float al[4], ah[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // selects, not products with zero: an unused O or buffer row may hold anything
                        const float o0 = __uint_as_float(r0[4 * v + e]), o1 = __uint_as_float(r1[4 * v + e]);
                        al[e] = (use_s ? svv[e] * cs : 0.f) + (u0l ? o0 * c0 : 0.f) + (u1l ? o1 * c1 : 0.f);
                        ah[e] = (u0h ? o0 * c0 : 0.f) + (u1h ? o1 * c1 : 0.f);
                    }
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        const int i = (4 * v + e) / 2;
                        of[i] = pack_bf16x2(w_loc * al[e] + w_hist * ah[e], w_loc * al[e + 1] + w_hist * ah[e + 1]);
                        ol[i] = pack_bf16x2(al[e], al[e + 1]);
                        oh[i] = pack_bf16x2(ah[e], ah[e + 1]);
                        orr[i] = pack_bf16x2(w_hist * (ah[e] - al[e]), w_hist * (ah[e + 1] - al[e + 1]));
                    }
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
            if (active && g == 0) {
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

// [rows, heads, 128] of 1-byte (int8) or 2-byte (bf16) elements; box = 128 bytes of one row of
// one head x 128 rows, 128-byte swizzle.
bool make_rows_map(CUtensorMap *m, const void *ptr, int rows, int heads, int esize) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)HD * esize, (cuuint64_t)heads * HD * esize};
    cuuint32_t box[3] = {(cuuint32_t)(128 / esize), 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kI8>
cudaError_t launch_2g(const AttnArgs &a, const float *q_scale, const float *k_scale, cudaStream_t s) {
    using L = Layout<kI8>;
    if (a.n_q == 0) return cudaSuccess;
    if (a.head_dim != HD) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    const void *kp = a.n_kv > 0 ? a.k : a.q;
    const void *vp = a.n_kv > 0 ? a.v : a.q;
    const int kv_rows = a.n_kv > 0 ? a.n_kv : a.n_q;
    if (!make_rows_map(&mq, a.q, a.n_q, a.heads, L::kQKElem) || !make_rows_map(&mk, kp, kv_rows, a.heads, L::kQKElem) ||
        !make_rows_map(&mv, vp, kv_rows, a.heads, 2))
        return cudaErrorInvalidValue;
    Split2gParams p;
    p.o_full = a.o_full; p.lse_full = a.lse_full;
    p.o_loc = a.o_loc; p.lse_loc = a.lse_loc;
    p.o_hist = a.o_hist; p.lse_hist = a.lse_hist;
    p.a_ops = a.a_loc_ops; p.r_ops = a.r_ops;
    p.n_q = a.n_q; p.heads = a.heads;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.segs.count = 0;
    for (int part = 0; part < 2; ++part)
        for (int i = 0; i < a.segs.count; ++i)
            if (a.segs.seg[i].part == part) p.segs.seg[p.segs.count++] = a.segs.seg[i];
    if (p.segs.count != a.segs.count) return cudaErrorInvalidValue;
    p.err_flag = a.err_flag;
    // K blocks are numbered in row order: each segment's first block index
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.n_blocks = 0;
    for (int i = 0; i < p.segs.count; ++i) {
        int first = 0;
        for (int j = 0; j < p.segs.count; ++j)
            if (p.segs.seg[j].begin < p.segs.seg[i].begin)
                first += (p.segs.seg[j].end - p.segs.seg[j].begin + kBlockN - 1) / kBlockN;
        p.seg_block0[i] = first;
        p.n_blocks += (p.segs.seg[i].end - p.segs.seg[i].begin + kBlockN - 1) / kBlockN;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_split_2g_kernel<kI8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits until the registers it asks for are free in the CTA's own
    // allocation: refuse to launch unless the split fits what the kernel is launched with
    static int launch_regs = -1;
    if (launch_regs < 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, attn_split_2g_kernel<kI8>);
        if (e != cudaSuccess) return e;
        launch_regs = fa.numRegs;
    }
    if (launch_regs * kThreads < kRegsNeeded) return cudaErrorInvalidConfiguration;
    dim3 grid((a.n_q + kBlockM - 1) / kBlockM, a.heads);
    attn_split_2g_kernel<kI8><<<grid, kThreads, L::kSmem, s>>>(mq, mk, mv, p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace

// head_dim 128 only.
cudaError_t launch_attn_bf16_2g(const AttnArgs &a, cudaStream_t s) { return launch_2g<false>(a, nullptr, nullptr, s); }

// int8 Q and K (a.q, a.k) with their scales, bf16 V; head_dim 128 only.
cudaError_t launch_attn_i8_2g(const AttnArgs &a, const float *q_scale, const float *k_scale, cudaStream_t s) {
    return launch_2g<true>(a, q_scale, k_scale, s);
}

}  // namespace ispa
