// Shared definitions of the libispa CUDA sources (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/ispa.h"

namespace ispa {

typedef __nv_bfloat16 bf16;

constexpr int kMaxBatch = 48;      // layers per batched launch of the solve kernels
constexpr int kMaxSegments = 6;    // KV row segments of one attention call

// A run of KV rows [begin, end) that belongs to one partition (0 = local, 1 = history).
struct Segment {
    int begin, end, part;
};

struct SegmentList {
    Segment seg[kMaxSegments];
    int count;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// Process-wide count of kernel launches made by the library (read by ispa_kernel_launches).
void note_launch();

// Latch a device-side error code (first writer wins) into the per-device flag.
__device__ __forceinline__ void raise_device_error(int *flag, int code) {
    if (flag) atomicCAS(flag, 0, code);
}

// ---- launchers implemented in the .cu files ------------------------------------------

struct AttnArgs {
    const void *q, *k, *v;
    void *o_full;
    float *lse_full;
    void *o_loc;
    float *lse_loc;
    void *o_hist;
    float *lse_hist;
    void *a_loc_ops;   // statistics operand A_loc [n_q, D] (bf16 or fp32), or null
    void *r_ops;       // statistics operand R [n_q, D], or null
    int n_q, n_kv, heads, head_dim;
    float scale;
    SegmentList segs;
    int *err_flag;
};

cudaError_t launch_attn_simt_f32(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attn_simt_bf16(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attn_bf16(const AttnArgs &a, cudaStream_t s);   // tcgen05 path
cudaError_t launch_attn_bf16_2sm(const AttnArgs &a, cudaStream_t s);   // tcgen05 CTA-pair path, head_dim 128
cudaError_t launch_attn_bf16_2g(const AttnArgs &a, cudaStream_t s);    // tcgen05, two softmax groups, head_dim 128
// int8 Q/K (a.q, a.k; scales [n_q][heads] and [heads][K blocks]), bf16 V; head_dim 128
cudaError_t launch_attn_i8_2g(const AttnArgs &a, const float *q_scale, const float *k_scale, cudaStream_t s);

// Batched SIMT GEMM: C_z[m][n] = alpha * sum_k A_z(m,k) B_z(k,n) + beta * C_z[m][n].
// A_z(m,k) = A[m*lda + k] if a_kcontig else A[k*lda + m]; B_z(k,n) = B[n*ldb + k] if
// b_kcontig else B[k*ldb + n]. lower_only restricts the update to tiles touching m >= n.
enum class ElemType { F32 = 0, BF16 = 1 };
struct GemmBatch {
    const void *A[kMaxBatch];
    const void *B[kMaxBatch];
    void *C[kMaxBatch];
};
struct GemmDesc {
    int M, N, K;
    int lda, ldb, ldc;
    bool a_kcontig, b_kcontig;
    ElemType a_type, b_type, c_type;
    float alpha, beta;
    bool lower_only;
    int batch;
};
cudaError_t launch_gemm_simt(const GemmDesc &d, const GemmBatch &b, cudaStream_t s);

// Ridge statistics from bf16 operands [n, D] row-major, float32 G/C/H updated in place.
cudaError_t launch_stats_bf16_layers(const void *a_loc, const void *r, int layers, int n, int D, float *const *G,
                                     float *const *C, float *const *H, int *err_flag, cudaStream_t s);
cudaError_t launch_stats_bf16(const void *a_loc, const void *r, int n, int D, float *G, float *C,
                               float *H, int *err_flag, cudaStream_t s);

// y[M][N] = A[M][K] W[K][N], bf16 in and out, tensor cores (gemm_bf16_sm100.cu).
cudaError_t launch_gemm_bf16(const void *A, const void *W, void *y, int M, int N, int K, int *err_flag,
                             cudaStream_t s);

// W8A8 projection (w8a8_sm100.cu): weights [K][N] -> int8 [N][K] + column scales; then
// y[M][N] (bf16) from activations A [M][K] (bf16) quantised by rows into q_a / s_a.
cudaError_t launch_quant_q_i8(const void *q, int n, int heads, int8_t *q8, float *q_scale, cudaStream_t s);
cudaError_t launch_quant_k_i8(const void *k, int heads, const SegmentList &segs, int n_blocks, int8_t *k8,
                              float *k_scale, cudaStream_t s);
cudaError_t launch_quant_cols(const void *w, ElemType t, int K, int N, int8_t *qt, float *scale, cudaStream_t s);
cudaError_t launch_project_w8a8(const void *A, int M, int K, const int8_t *qt, const float *col_scale, int N,
                                void *y, int8_t *q_a, float *s_a, int *err_flag, cudaStream_t s);

// Solve-phase kernels (float32, batched over layers).
struct PtrBatch {
    void *p[kMaxBatch];
};

// M = G + lambda I = L L^T and X = L^-1 into P, float32, one cluster of CTAs per layer
// (chol_inv_sm100.cu); status[z] = ISPA_ERR_NOT_SPD on a non-positive pivot.
cudaError_t launch_chol_inv(const PtrBatch &G, const PtrBatch &M, const PtrBatch &P, int D, float lambda, int batch,
                            int *status, cudaStream_t s);
// The same for an n x n diagonal block already in M (pointers at the block, row stride ld): its
// L^-1 into the matching block of P.
cudaError_t launch_chol_inv_block(const PtrBatch &M, const PtrBatch &P, int n, int ld, int batch, int *status,
                                  cudaStream_t s);

// 3xTF32 tensor-core GEMM for D x D products (gemm_tf32_sm100.cu).
// Source row stride ld (0: cols); destination entries dst_bstride elements apart (0: rows*cols).
cudaError_t launch_split_tf32(const PtrBatch &src, ElemType t, float *hi, float *lo, int rows, int cols,
                              bool transpose, int batch, cudaStream_t s, size_t ld = 0, size_t dst_bstride = 0);
struct Tf32Opts {
    int a_tri = 0;                      // 1: A lower triangular, 2: A upper triangular (M = K)
    bool sym = false;                   // B is A: only output tiles on and below the diagonal
    const PtrBatch *dot_x = nullptr;    // trace partials against X (float32 or bf16)
    bool dot_x_bf16 = false;
    double *dot_out = nullptr;
    const PtrBatch *dot_x2 = nullptr;   // a second float32 X
    double *dot_out2 = nullptr;
    float *split_hi = nullptr;          // C's TF32 split (hi, lo), [batch][M][N] or transposed
    float *split_lo = nullptr;
    bool split_t = false;
    size_t split_bstride = 0;           // 0: M*N
    size_t ldc = 0, c_bstride = 0;      // C's row and batch strides (0: N, M*N)
    bool c_sub = false;                 // C = C - A B
    bool write_c = true;
};
cudaError_t launch_gemm_tf32x3(const float *Ah, const float *Al, const float *Bh, const float *Bl, float *C, int M,
                               int N, int K, int batch, int *err_flag, cudaStream_t s, const Tf32Opts &o = Tf32Opts());

}  // namespace ispa
