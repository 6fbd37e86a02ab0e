// Cholesky factor and explicit inverse of an n x n symmetric positive definite matrix in one
// launch, one thread-block cluster of kCL CTAs per layer [ISPA §3.2: the ridge system
// (G + lambda I) dW = C W]: either the whole M = G + lambda I (n = D), or one diagonal block of the
// blocked factorisation in solve.cu, whose inverse is the matching diagonal block of L^-1.
//
// The cluster walks the 64-wide block columns k of M (right-looking); per step two phases, each
// closed by a cluster barrier:
//   A  every CTA factors the diagonal block in registers (the same arithmetic in every CTA, so
//      the same bits) and inverts it into T = L_kk^-1 in shared memory; then the CTAs share the
//      jobs  L_ik = A_ik T^T  (i > k, the panel)  and  X_kc = T B_kc  (c < k, block row k of
//      X = L^-1; X_kk = T).
//   B  the CTAs share the trailing updates  A_ij -= L_ik L_jk^T  (k < j <= i)  and the
//      substitution updates  B_ic -= L_ik X_kc  (i > k, c <= k).
// B starts as I (L X = I solved by block forward substitution), so after the last step P holds
// X = L^-1 with zeros above the diagonal. Every job is one 64 x 64 x 64 product on the CUDA
// cores (256 threads, 4 x 4 outputs each, float32), its operand panels staged in shared memory
// by cp.async and prefetched one job ahead. M and P are shared by the cluster through L2: every
// load that may see another CTA's write bypasses L1 (cp.async.cg, ld.global.cg) and the
// barriers are release/acquire at cluster scope after a device-scope fence.
//
// The whole chain is 2 * n/64 cluster barriers and no kernel boundaries; the layers' clusters
// are independent. A non-positive pivot marks the layer ISPA_ERR_NOT_SPD; the NaN it produces
// runs through L and X (no trap, no early exit: every CTA takes every barrier).
#include "common.cuh"

namespace ispa {
namespace {

constexpr int kCL = 8;            // CTAs per layer (portable cluster size)
constexpr int kNB = 64;           // block size
constexpr int kLd = 68;           // row stride of a staged 64 x 64 panel (floats): 16-byte rows, spread banks
constexpr int kThreads = 256;
constexpr int kPanel = kNB * kLd;
// shared memory (floats): T, the factored block Lf, two double-buffered operand pairs, 1/L_jj
constexpr int kOffT = 0;
constexpr int kOffLf = kOffT + kPanel;
constexpr int kOffBuf = kOffLf + kNB * (kNB + 1);
constexpr int kOffInv = kOffBuf + 4 * kPanel;
constexpr int kSmemFloats = kOffInv + kNB + 2 * kNB;
constexpr int kSmemBytes = kSmemFloats * 4;

__device__ __forceinline__ void cluster_sync_rel_acq() {
    __threadfence();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// 64 x 64 block (r, c) of a D x D row-major matrix into a [64][kLd] panel
__device__ __forceinline__ void stage_panel(float *dst, const float *Mz, int D, int r, int c) {
    const float *src = Mz + (size_t)r * kNB * D + (size_t)c * kNB;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int idx = threadIdx.x + u * kThreads;   // 1024 16-byte pieces
        const int row = idx >> 4, col = (idx & 15) * 4;
        cp_async16(dst + row * kLd + col, src + (size_t)row * D + col);
    }
}

// The jobs. kind 0: M(i,j) -= M(i,k) M(j,k)^T; 1: P(i,j) -= M(i,k) P(k,j);
// 2: M(i,k) = M(i,k) T^T; 3: P(k,j) = T P(k,j).
struct Job {
    int kind, i, j;
};

// Phase A's jobs of step k: the panel (i = k+1 .. nb-1), then block row k of X (c = 0 .. k-1).
__device__ __forceinline__ Job job_a(int t, int k, int nb) {
    const int m = nb - 1 - k;
    if (t < m) return {2, k + 1 + t, k};
    return {3, k, t - m};
}

// Phase B's jobs of step k: the trailing lower triangle (row-major), then rows i > k of X.
__device__ __forceinline__ Job job_b(int t, int k, int nb) {
    const int m = nb - 1 - k;
    const int tri = m * (m + 1) / 2;
    if (t < tri) {
        int i = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
        while (i * (i + 1) / 2 > t) --i;
        while ((i + 1) * (i + 2) / 2 <= t) ++i;
        return {0, k + 1 + i, k + 1 + (t - i * (i + 1) / 2)};
    }
    const int u = t - tri;
    return {1, k + 1 + u / (k + 1), u % (k + 1)};
}

// Stage the global operand panels of a job into buffer pair `buf` (A in slot 0, B in slot 1).
__device__ __forceinline__ void stage_job(const Job &jb, int k, float *bufs, float *Mz, float *Pz, int D) {
    float *sa = bufs, *sb = bufs + kPanel;
    switch (jb.kind) {
        case 0: stage_panel(sa, Mz, D, jb.i, k); stage_panel(sb, Mz, D, jb.j, k); break;
        case 1: stage_panel(sa, Mz, D, jb.i, k); stage_panel(sb, Pz, D, k, jb.j); break;
        case 2: stage_panel(sa, Mz, D, jb.i, k); break;
        default: stage_panel(sb, Pz, D, k, jb.j); break;
    }
}

// acc[a][b] = sum_q A[ty + 16a][q] * B(q, tx + 16b); B(q, n) = Bs[n][q] (TN) or Bs[q][n] (NN).
template <bool NN>
__device__ __forceinline__ void panel_product(const float *As, const float *Bs, float acc[4][4], int tx, int ty) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
    for (int q = 0; q < kNB; q += 4) {
        float4 av[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) av[a] = *reinterpret_cast<const float4 *>(As + (ty + 16 * a) * kLd + q);
        float bv[4][4];   // [q offset][b]
        if (NN) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int b = 0; b < 4; ++b) bv[e][b] = Bs[(q + e) * kLd + tx + 16 * b];
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const float4 w = *reinterpret_cast<const float4 *>(Bs + (tx + 16 * b) * kLd + q);
                bv[0][b] = w.x; bv[1][b] = w.y; bv[2][b] = w.z; bv[3][b] = w.w;
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float ae[4] = {av[a].x, av[a].y, av[a].z, av[a].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(ae[e], bv[e][b], acc[a][b]);
        }
    }
}

__device__ __forceinline__ void run_job(const Job &jb, int k, const float *bufs, const float *Ts, float *Mz, float *Pz,
                                        int D) {
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const float *sa = bufs, *sb = bufs + kPanel;
    float *c = (jb.kind == 0 || jb.kind == 2 ? Mz : Pz) + (size_t)jb.i * kNB * D + (size_t)jb.j * kNB;
    // an update's old values are fetched before the product, so their latency hides behind it
    float old[4][4];
    if (jb.kind <= 1) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) old[a][b] = __ldcg(c + (size_t)(ty + 16 * a) * D + tx + 16 * b);
    }
    float acc[4][4];
    switch (jb.kind) {
        case 0: panel_product<false>(sa, sb, acc, tx, ty); break;
        case 1: panel_product<true>(sa, sb, acc, tx, ty); break;
        case 2: panel_product<false>(sa, Ts, acc, tx, ty); break;
        default: panel_product<true>(Ts, sb, acc, tx, ty); break;
    }
    const bool overwrite = jb.kind >= 2;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            __stcg(c + (size_t)(ty + 16 * a) * D + tx + 16 * b, overwrite ? acc[a][b] : old[a][b] - acc[a][b]);
}

// Run this CTA's share (t = rank, rank + kCL, ...) of n jobs, the next job's panels staged while
// the current one computes.
// The first job's panels are staged (and committed) by the caller.
template <bool PHASE_A>
__device__ __forceinline__ void stage_first(int n, int rank, int k, int nb, float *buf0, float *Mz, float *Pz, int D) {
    if (rank < n) stage_job(PHASE_A ? job_a(rank, k, nb) : job_b(rank, k, nb), k, buf0, Mz, Pz, D);
    cp_async_commit();
}

template <bool PHASE_A>
__device__ __forceinline__ void run_jobs(int n, int rank, int k, int nb, float *buf0, const float *Ts, float *Mz,
                                         float *Pz, int D) {
    int t = rank, cur = 0;
    for (; t < n; t += kCL) {
        const Job jb = PHASE_A ? job_a(t, k, nb) : job_b(t, k, nb);
        if (t + kCL < n)
            stage_job(PHASE_A ? job_a(t + kCL, k, nb) : job_b(t + kCL, k, nb), k, buf0 + (cur ^ 1) * 2 * kPanel, Mz,
                      Pz, D);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        run_job(jb, k, buf0 + cur * 2 * kPanel, Ts, Mz, Pz, D);
        __syncthreads();   // the buffer is restaged two jobs on
        cur ^= 1;
    }
    cp_async_wait0();
}

// Threads 0..63: factor the diagonal block (k, k) of M and write T = L_kk^-1 to Ts (row stride
// kLd). Returns true on a non-positive pivot. Kept out of line: the two 64-float rows then live
// in registers.
__device__ __noinline__ bool factor_invert_diag(const float *Mz, int D, int k, float *Lf, float *Ts, float *inv,
                                                float *col) {
    const int tid = threadIdx.x;
    bool bad = false;
    {
        // thread i holds row i of the block; column j: publish, one barrier among the 64 threads,
        // update the elements right of j (all of them: the upper part is never stored), scale a_ij
        float a[kNB];
        const float4 *row = reinterpret_cast<const float4 *>(Mz + (size_t)(k * kNB + tid) * D + k * kNB);
#pragma unroll
        for (int c = 0; c < kNB / 4; ++c) {
            const float4 v = __ldcg(row + c);
            a[4 * c] = v.x; a[4 * c + 1] = v.y; a[4 * c + 2] = v.z; a[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            float *cj = col + (j & 1) * kNB;
            cj[tid] = a[j];
            asm volatile("bar.sync 1, 64;" ::: "memory");
            const float d = cj[j];
            float rs = __int_as_float(0x7fc00000);
            if (d > 0.f) rs = rsqrtf(d);
            else bad = true;
            const float f = a[j] * (rs * rs);
#pragma unroll
            for (int c = j + 1; c < kNB; ++c) a[c] -= f * cj[c];
            a[j] = tid == j ? d * rs : a[j] * rs;
        }
#pragma unroll
        for (int c = 0; c < kNB; ++c) Lf[tid * (kNB + 1) + c] = c <= tid ? a[c] : 0.f;
        inv[tid] = 1.f / Lf[tid * (kNB + 1) + tid];
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    {
        // column tid of T: forward substitution on e_tid, each finished element subtracted at
        // once from the ones below
        float t[kNB];
#pragma unroll
        for (int i = 0; i < kNB; ++i) t[i] = i == tid ? 1.f : 0.f;
#pragma unroll
        for (int p = 0; p < kNB; ++p) {
            t[p] *= inv[p];
#pragma unroll
            for (int i = p + 1; i < kNB; ++i) t[i] -= Lf[i * (kNB + 1) + p] * t[p];
        }
#pragma unroll
        for (int i = 0; i < kNB; ++i) Ts[i * kLd + tid] = t[i];
    }
    return bad;
}

// FILL_M: M = G + lambda I first (the whole matrix, n = ld); otherwise M already holds the n x n
// block to factor (row stride ld). P (the same block of the inverse) is set to I either way.
template <bool FILL_M>
__global__ void __cluster_dims__(kCL, 1, 1) __launch_bounds__(kThreads, 2)
chol_inv_cluster_kernel(PtrBatch G, PtrBatch M, PtrBatch P, int n, int ld, float lambda, int *status) {
    extern __shared__ __align__(16) float sm[];
    float *Ts = sm + kOffT, *Lf = sm + kOffLf, *buf0 = sm + kOffBuf, *inv = sm + kOffInv;
    float *col = inv + kNB;   // [2][64]
    const int rank = (int)blockIdx.x;   // cluster of kCL along x: blockIdx.x is the rank
    const int z = blockIdx.y;
    float *Mz = static_cast<float *>(M.p[z]);
    float *Pz = static_cast<float *>(P.p[z]);
    const int nb = n / kNB;
    const int D = ld;   // row stride of M and P
    const int tid = threadIdx.x;

    // (M = G + lambda I,) P = I: each CTA writes its share of rows
    {
        const int r0 = (int)((long long)n * rank / kCL), r1 = (int)((long long)n * (rank + 1) / kCL);
        const int q = n / 4;
        for (long long idx = tid; idx < (long long)(r1 - r0) * q; idx += kThreads) {
            const int r = r0 + (int)(idx / q), c4 = (int)(idx % q) * 4;
            const int d = r - c4;
            const float4 e = make_float4(d == 0 ? 1.f : 0.f, d == 1 ? 1.f : 0.f, d == 2 ? 1.f : 0.f, d == 3 ? 1.f : 0.f);
            if (FILL_M) {
                const float *Gz = static_cast<const float *>(G.p[z]);
                float4 g = *reinterpret_cast<const float4 *>(Gz + (size_t)r * D + c4);
                g.x += d == 0 ? lambda : 0.f;
                g.y += d == 1 ? lambda : 0.f;
                g.z += d == 2 ? lambda : 0.f;
                g.w += d == 3 ? lambda : 0.f;
                __stcg(reinterpret_cast<float4 *>(Mz + (size_t)r * D + c4), g);
            }
            __stcg(reinterpret_cast<float4 *>(Pz + (size_t)r * D + c4), e);
        }
    }
    cluster_sync_rel_acq();

    bool bad = false;
    for (int k = 0; k < nb; ++k) {
        const int m = nb - 1 - k;
        // ---- phase A: factor and invert the diagonal block (every CTA), then the panel and
        // block row k of X (the first job's panel is fetched meanwhile)
        stage_first<true>(m + k, rank, k, nb, buf0, Mz, Pz, D);
        if (tid < kNB) bad |= factor_invert_diag(Mz, D, k, Lf, Ts, inv, col);
        __syncthreads();
        if (rank == 0) {
            // X_kk = T
            float *xk = Pz + (size_t)k * kNB * D + (size_t)k * kNB;
            for (int idx = tid; idx < kNB * kNB; idx += kThreads)
                __stcg(xk + (size_t)(idx >> 6) * D + (idx & 63), Ts[(idx >> 6) * kLd + (idx & 63)]);
        }
        run_jobs<true>(m + k, rank, k, nb, buf0, Ts, Mz, Pz, D);
        cluster_sync_rel_acq();
        // ---- phase B: trailing update and the substitution updates
        const int nbj = m * (m + 1) / 2 + m * (k + 1);
        stage_first<false>(nbj, rank, k, nb, buf0, Mz, Pz, D);
        run_jobs<false>(nbj, rank, k, nb, buf0, Ts, Mz, Pz, D);
        cluster_sync_rel_acq();
    }
    if (bad && rank == 0 && tid == 0) status[z] = ISPA_ERR_NOT_SPD;
}

}  // namespace

// M = G + lambda I; X = L^-1 into P (L L^T = M), for `batch` layers of D x D float32 (D a
// multiple of 64). M and P are scratch (M ends holding the unfactored diagonal blocks and L
// below them; P is X, zero above the diagonal).
cudaError_t launch_chol_inv(const PtrBatch &G, const PtrBatch &M, const PtrBatch &P, int D, float lambda, int batch,
                            int *status, cudaStream_t s) {
    if (D % kNB || batch <= 0 || batch > kMaxBatch) return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(chol_inv_cluster_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    chol_inv_cluster_kernel<true><<<dim3(kCL, batch), kThreads, kSmemBytes, s>>>(G, M, P, D, D, lambda, status);
    note_launch();
    return cudaGetLastError();
}

// The same for an n x n diagonal block already in M (pointers at the block, row stride ld):
// its L^-1 into the matching block of P (M's block is overwritten as scratch).
cudaError_t launch_chol_inv_block(const PtrBatch &M, const PtrBatch &P, int n, int ld, int batch, int *status,
                                  cudaStream_t s) {
    if (n % kNB || ld % 4 || n > ld || batch <= 0 || batch > kMaxBatch) return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(chol_inv_cluster_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    chol_inv_cluster_kernel<false><<<dim3(kCL, batch), kThreads, kSmemBytes, s>>>(M, M, P, n, ld, 0.f, status);
    note_launch();
    return cudaGetLastError();
}

}  // namespace ispa
