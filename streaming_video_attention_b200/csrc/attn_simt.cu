// Split (decomposable) attention on the CUDA cores, float32 arithmetic.
//
// [ISPA §3.1 step 1, §3.4]: one pass over the KV rows keeps two online-softmax states,
// one for the local partition (sink frame + current chunk) and one for the history
// partition, and merges them by their log-sum-exps. This kernel serves the float32
// workloads, where the tolerance rules out bf16 tensor-core operands; every
// product and sum is a float32 FMA.
//
// Mapping: one CTA = 128 threads = (128 / TPQ) query rows of one head; TPQ = head_dim/64
// threads share a query row, each owning 64 of its dimensions (q, and two output
// accumulators, live in registers). KV rows stream through shared memory 32 at a time.
#include "common.cuh"

namespace ispa {
namespace {

constexpr int kThreads = 128;
constexpr int kKeyTile = 32;

template <typename T, int DH>
__global__ void __launch_bounds__(kThreads) attn_split_simt_kernel(AttnArgs a) {
    constexpr int TPQ = DH / 64;
    constexpr int QPB = kThreads / TPQ;
    __shared__ float Ks[kKeyTile][DH];
    __shared__ float Vs[kKeyTile][DH];

    const int h = blockIdx.y;
    const int qi = blockIdx.x * QPB + threadIdx.x / TPQ;
    const int sub = threadIdx.x % TPQ;
    const bool active = qi < a.n_q;
    const int H = a.heads;
    const T *Q = static_cast<const T *>(a.q);
    const T *Kp = static_cast<const T *>(a.k);
    const T *Vp = static_cast<const T *>(a.v);

    float q[64];
#pragma unroll
    for (int c = 0; c < 64; ++c)
        q[c] = active ? to_f32(Q[((size_t)qi * H + h) * DH + sub * 64 + c]) : 0.f;

    float a_loc[64], acc[64];
    float lse_loc = -INFINITY, lse_hist = -INFINITY;

    for (int part = 0; part < 2; ++part) {
        float m = -INFINITY, l = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.f;
        for (int si = 0; si < a.segs.count; ++si) {
            const Segment sg = a.segs.seg[si];
            if (sg.part != part) continue;
            for (int t0 = sg.begin; t0 < sg.end; t0 += kKeyTile) {
                const int nt = min(kKeyTile, sg.end - t0);
                __syncthreads();
                for (int idx = threadIdx.x; idx < nt * DH; idx += kThreads) {
                    const int r = idx / DH, c = idx % DH;
                    const size_t g = ((size_t)(t0 + r) * H + h) * DH + c;
                    Ks[r][c] = to_f32(Kp[g]);
                    Vs[r][c] = to_f32(Vp[g]);
                }
                __syncthreads();
                for (int j = 0; j < nt; ++j) {
                    float s = 0.f;
#pragma unroll
                    for (int c = 0; c < 64; ++c) s = fmaf(q[c], Ks[j][sub * 64 + c], s);
                    if (TPQ == 2) s += __shfl_xor_sync(0xffffffffu, s, 1);
                    s *= a.scale;
                    if (s > m) {
                        const float corr = expf(m - s);
                        l = fmaf(l, corr, 1.f);
#pragma unroll
                        for (int c = 0; c < 64; ++c) acc[c] = fmaf(acc[c], corr, Vs[j][sub * 64 + c]);
                        m = s;
                    } else {
                        const float p = expf(s - m);
                        l += p;
#pragma unroll
                        for (int c = 0; c < 64; ++c) acc[c] = fmaf(p, Vs[j][sub * 64 + c], acc[c]);
                    }
                }
            }
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse = l > 0.f ? m + logf(l) : -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] *= inv;
        if (part == 0) {
            lse_loc = lse;
#pragma unroll
            for (int c = 0; c < 64; ++c) a_loc[c] = acc[c];
        } else {
            lse_hist = lse;
        }
    }
    if (!active) return;

    // acc now holds A_hist. Merge the two partitions by their log-sum-exps.
    const float mx = fmaxf(lse_loc, lse_hist);
    float lse_full, w_loc, w_hist;
    if (mx == -INFINITY) {
        lse_full = -INFINITY; w_loc = 0.f; w_hist = 0.f;
    } else {
        const float el = expf(lse_loc - mx), eh = expf(lse_hist - mx);
        lse_full = mx + logf(el + eh);
        w_loc = el / (el + eh);
        w_hist = eh / (el + eh);
    }
    const size_t obase = ((size_t)qi * H + h) * DH + sub * 64;
    T *Of = static_cast<T *>(a.o_full);
#pragma unroll
    for (int c = 0; c < 64; ++c) Of[obase + c] = from_f32<T>(w_loc * a_loc[c] + w_hist * acc[c]);
    if (a.o_loc) {
        T *Ol = static_cast<T *>(a.o_loc);
#pragma unroll
        for (int c = 0; c < 64; ++c) Ol[obase + c] = from_f32<T>(a_loc[c]);
    }
    if (a.o_hist) {
        T *Oh = static_cast<T *>(a.o_hist);
#pragma unroll
        for (int c = 0; c < 64; ++c) Oh[obase + c] = from_f32<T>(acc[c]);
    }
    if (a.a_loc_ops) {
        // Statistics operands: A_loc and R = A_full - A_loc = w_hist (A_hist - A_loc),
        // rounded once to the operand type.
        T *Ao = static_cast<T *>(a.a_loc_ops);
        T *Ro = static_cast<T *>(a.r_ops);
        const size_t D = (size_t)H * DH;
        const size_t base = (size_t)qi * D + (size_t)h * DH + sub * 64;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
            Ao[base + c] = from_f32<T>(a_loc[c]);
            Ro[base + c] = from_f32<T>(w_hist * (acc[c] - a_loc[c]));
        }
    }
    if (sub == 0) {
        a.lse_full[(size_t)h * a.n_q + qi] = lse_full;
        if (a.lse_loc) a.lse_loc[(size_t)h * a.n_q + qi] = lse_loc;
        if (a.lse_hist) a.lse_hist[(size_t)h * a.n_q + qi] = lse_hist;
    }
}

template <typename T>
cudaError_t launch_simt(const AttnArgs &a, cudaStream_t s) {
    if (a.n_q == 0) return cudaSuccess;
    if (a.head_dim == 64) {
        dim3 grid((a.n_q + kThreads - 1) / kThreads, a.heads);
        attn_split_simt_kernel<T, 64><<<grid, kThreads, 0, s>>>(a); note_launch();
    } else if (a.head_dim == 128) {
        dim3 grid((a.n_q + kThreads / 2 - 1) / (kThreads / 2), a.heads);
        attn_split_simt_kernel<T, 128><<<grid, kThreads, 0, s>>>(a); note_launch();
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt_f32(const AttnArgs &a, cudaStream_t s) { return launch_simt<float>(a, s); }
cudaError_t launch_attn_simt_bf16(const AttnArgs &a, cudaStream_t s) { return launch_simt<bf16>(a, s); }

}  // namespace ispa
