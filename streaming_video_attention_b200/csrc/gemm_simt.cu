// Batched float32 GEMM on the CUDA cores, used where float32 products are required:
// the statistics of the float32 workloads and the float32 absorb solve (Y = C W, the
// trailing updates of the blocked Cholesky factorisation and of the triangular solves,
// and the products G dW, G W, H W of the reconstruction error).
//
// C_z = alpha * op(A_z) op(B_z) + beta * C_z, one 128x128 output tile per CTA, 256
// threads with 8x8 outputs each, k in steps of 8 through double-buffered shared memory.
// Each output element is reduced in a fixed order (no atomics), so results repeat bit
// for bit.
#include "common.cuh"

namespace ispa {
namespace {

constexpr int BM = 128, BN = 128, BKT = 8, PAD = 4;

template <typename T>
__device__ __forceinline__ float ld(const T *p, size_t i) { return to_f32(p[i]); }

template <typename TA, typename TB, typename TC, bool AK, bool BKC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc d, GemmBatch b) {
    const int z = blockIdx.z;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    if (d.lower_only && n0 > m0 + BM - 1) return;
    const TA *A = static_cast<const TA *>(b.A[z]);
    const TB *B = static_cast<const TB *>(b.B[z]);
    TC *C = static_cast<TC *>(b.C[z]);

    __shared__ __align__(16) float As[2][BKT][BM + PAD];
    __shared__ __align__(16) float Bs[2][BKT][BN + PAD];

    const int t = threadIdx.x;
    float ra[4], rb[4];

    auto load_regs = [&](int k0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int mm, kk;
            if (AK) { kk = t % BKT; mm = t / BKT + 32 * i; }
            else    { mm = t % BM;  kk = t / BM + 2 * i; }
            const int gm = m0 + mm, gk = k0 + kk;
            float v = 0.f;
            if (gm < d.M && gk < d.K)
                v = AK ? ld(A, (size_t)gm * d.lda + gk) : ld(A, (size_t)gk * d.lda + gm);
            ra[i] = v;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int nn, kk;
            if (BKC) { kk = t % BKT; nn = t / BKT + 32 * i; }
            else     { nn = t % BN;  kk = t / BN + 2 * i; }
            const int gn = n0 + nn, gk = k0 + kk;
            float v = 0.f;
            if (gn < d.N && gk < d.K)
                v = BKC ? ld(B, (size_t)gn * d.ldb + gk) : ld(B, (size_t)gk * d.ldb + gn);
            rb[i] = v;
        }
    };
    auto store_smem = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int mm, kk;
            if (AK) { kk = t % BKT; mm = t / BKT + 32 * i; }
            else    { mm = t % BM;  kk = t / BM + 2 * i; }
            As[buf][kk][mm] = ra[i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int nn, kk;
            if (BKC) { kk = t % BKT; nn = t / BKT + 32 * i; }
            else     { nn = t % BN;  kk = t / BN + 2 * i; }
            Bs[buf][kk][nn] = rb[i];
        }
    };

    const int tx = t % 16, ty = t / 16;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    const int nk = (d.K + BKT - 1) / BKT;
    if (nk > 0) {
        load_regs(0);
        store_smem(0);
    }
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) load_regs((kt + 1) * BKT);
#pragma unroll
        for (int kk = 0; kk < BKT; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (kt + 1 < nk) store_smem(buf ^ 1);
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (gm >= d.M) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
            if (gn >= d.N) continue;
            const size_t idx = (size_t)gm * d.ldc + gn;
            float v = d.alpha * acc[i][j];
            if (d.beta != 0.f) v = fmaf(d.beta, to_f32(C[idx]), v);
            C[idx] = from_f32<TC>(v);
        }
    }
}

template <typename TA, typename TB, typename TC>
cudaError_t dispatch_layout(const GemmDesc &d, const GemmBatch &b, cudaStream_t s) {
    dim3 grid((d.N + BN - 1) / BN, (d.M + BM - 1) / BM, d.batch);
    if (d.a_kcontig && d.b_kcontig) { gemm_simt_kernel<TA, TB, TC, true, true><<<grid, 256, 0, s>>>(d, b); note_launch(); }
    else if (d.a_kcontig)           { gemm_simt_kernel<TA, TB, TC, true, false><<<grid, 256, 0, s>>>(d, b); note_launch(); }
    else if (d.b_kcontig)           { gemm_simt_kernel<TA, TB, TC, false, true><<<grid, 256, 0, s>>>(d, b); note_launch(); }
    else                            { gemm_simt_kernel<TA, TB, TC, false, false><<<grid, 256, 0, s>>>(d, b); note_launch(); }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmDesc &d, const GemmBatch &b, cudaStream_t s) {
    if (d.M <= 0 || d.N <= 0 || d.batch <= 0) return cudaSuccess;
    if (d.batch > kMaxBatch) return cudaErrorInvalidValue;
    const bool abf = d.a_type == ElemType::BF16, bbf = d.b_type == ElemType::BF16;
    if (d.c_type == ElemType::BF16) {
        if (d.beta != 0.f) return cudaErrorInvalidValue;
        if (abf && bbf) return dispatch_layout<bf16, bf16, bf16>(d, b, s);
        if (abf)        return dispatch_layout<bf16, float, bf16>(d, b, s);
        if (bbf)        return dispatch_layout<float, bf16, bf16>(d, b, s);
        return dispatch_layout<float, float, bf16>(d, b, s);
    }
    if (abf && bbf) return dispatch_layout<bf16, bf16, float>(d, b, s);
    if (abf)        return dispatch_layout<bf16, float, float>(d, b, s);
    if (bbf)        return dispatch_layout<float, bf16, float>(d, b, s);
    return dispatch_layout<float, float, float>(d, b, s);
}

}  // namespace ispa
