// Absorb solve and reconstruction error, float32, batched over layers
// [ISPA §3.1 step 2, §3.2, §3.3, §4.1 "Eq. 5"].
//
//   with D a multiple of 128:
//   Y = C W                                   3xTF32 product (gemm_tf32_sm100.cu)
//   M = G + lambda I = L L^T, X = L^-1        blocked by 512 (256, 128) columns: each diagonal
//                                             block factored and inverted by a thread-block
//                                             cluster per layer (chol_inv_sm100.cu); the panel,
//                                             the trailing update and the rows of X as 3xTF32
//                                             products (chol_inv_blocked)
//   dW = X^T X (C W)                          Z = X (C W), dW = X^T Z on the tensor cores
//                                             (3xTF32, the zero triangle of X skipped)
//   otherwise:
//   M = G + lambda I                          fill_shifted
//   M = L L^T (blocked, right-looking)        potrf_diag + trsm_panel + GEMM trailing update
//   dW = L^-T L^-1 (C W)                      trsv_block + GEMM per block, both ways, on
//                                             (C W) itself
//   five traces -> E^2, T^2, eps              tensor cores: the Gram products W W^T and
//                                             dW dW^T (lower tiles only) dotted with G and H,
//                                             and tr(W^T C W), tr(dW^T C W), in the GEMM
//                                             epilogues; otherwise GEMMs G dW, H W, G W, then
//                                             dot_partials
//
// On the CUDA-core path the block size is 64 (D must be a multiple of 64): each 64 x 64
// diagonal block is factored (potrf_diag) and each panel below it solved (trsm_panel) by CTAs
// whose threads hold one row of the block in registers, and everything of order D^3 runs in
// batched GEMMs. A non-positive pivot marks the layer ISPA_ERR_NOT_SPD and turns its results to
// NaN; nothing traps.
#include "common.cuh"

namespace ispa {
namespace {

constexpr int NB = 64;

__global__ void fill_shifted_kernel(PtrBatch src, PtrBatch dst, int D, float lambda) {
    const int z = blockIdx.y;
    const float *S = static_cast<const float *>(src.p[z]);
    float *Dst = static_cast<float *>(dst.p[z]);
    const size_t n = (size_t)D * D;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float v = S[i];
        if (i / D == i % D) v += lambda;
        Dst[i] = v;
    }
}

// Cholesky factor of the NB x NB diagonal block at (k0, k0), in place (lower triangle). One
// CTA of NB threads per layer; thread i holds row i of the block in registers (the column loop
// is unrolled so that every index is a constant). Column j: each row publishes its element of
// column j (double-buffered, so one barrier per column), then every row reads the pivot d,
// subtracts a_ij a_kj / d from its elements k in (j, i] and scales its own a_ij by 1/sqrt(d)
// (L_ij = a_ij / sqrt(d), L_jj = d / sqrt(d)).
__global__ void __launch_bounds__(NB) potrf_diag_kernel(PtrBatch M, int D, int k0, int *status) {
    __shared__ float col[2][NB];
    const int z = blockIdx.x;
    float *Mz = static_cast<float *>(M.p[z]);
    const int i = threadIdx.x;
    float a[NB];
    const float *row = Mz + (size_t)(k0 + i) * D + k0;
#pragma unroll
    for (int c = 0; c < NB; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(row + c);
        a[c] = v.x; a[c + 1] = v.y; a[c + 2] = v.z; a[c + 3] = v.w;
    }
    bool bad = false;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        float *cj = col[j & 1];
        if (i >= j) cj[i] = a[j];
        __syncthreads();
        const float d = cj[j];
        float rs = __int_as_float(0x7fc00000);
        if (d > 0.f) rs = rsqrtf(d);
        else bad = true;
        if (i > j) {
            const float f = a[j] * (rs * rs);
#pragma unroll
            for (int k = j + 1; k < NB; ++k)
                if (k <= i) a[k] -= f * cj[k];
            a[j] *= rs;
        } else if (i == j) {
            a[j] = d * rs;
        }
    }
    if (bad && i == 0) status[z] = ISPA_ERR_NOT_SPD;
    float *out = Mz + (size_t)(k0 + i) * D + k0;
#pragma unroll
    for (int c = 0; c < NB; ++c)
        if (c <= i) out[c] = a[c];
}

// Rows below the diagonal block: L21 = A21 L11^-T. One CTA of NB threads per NB rows; thread i
// holds its row of A21 in registers (unrolled loops, constant indices) and substitutes forward
// column by column, each finished element x_j (times 1/L_jj) subtracted at once from the later
// ones (x_c -= x_j L_cj), so the dependent chain is one multiply and one FMA per column. The
// factored diagonal block and its reciprocal pivots sit in shared memory, read by broadcast.
__global__ void __launch_bounds__(NB) trsm_panel_kernel(PtrBatch M, int D, int k0) {
    __shared__ __align__(16) float Lk[NB][NB];
    __shared__ float inv[NB];
    const int z = blockIdx.y;
    float *Mz = static_cast<float *>(M.p[z]);
    const int i = threadIdx.x;
    const int r = k0 + NB + blockIdx.x * NB + i;
    // column i of the diagonal block: coalesced reads, conflict-free stores
    for (int rr = 0; rr < NB; ++rr) Lk[rr][i] = i <= rr ? Mz[(size_t)(k0 + rr) * D + k0 + i] : 0.f;
    inv[i] = 1.f / Mz[(size_t)(k0 + i) * D + k0 + i];
    float x[NB];
    if (r < D) {
        const float *row = Mz + (size_t)r * D + k0;
#pragma unroll
        for (int c = 0; c < NB; c += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(row + c);
            x[c] = v.x; x[c + 1] = v.y; x[c + 2] = v.z; x[c + 3] = v.w;
        }
    }
    __syncthreads();
    if (r >= D) return;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        x[j] *= inv[j];
#pragma unroll
        for (int c = j + 1; c < NB; ++c) x[c] -= x[j] * Lk[c][j];
    }
    float *out = Mz + (size_t)r * D + k0;
#pragma unroll
    for (int c = 0; c < NB; c += 4) *reinterpret_cast<float4 *>(out + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
}

// X_k = L_kk^-1 X_k (forward) or L_kk^-T X_k (backward) for the NB rows of block k,
// every column of X at once (one thread per column); each finished element (times the
// reciprocal pivot) is subtracted at once from the elements still to come.
template <bool TRANS>
__global__ void __launch_bounds__(128) trsv_block_kernel(PtrBatch L, PtrBatch X, int D, int k0) {
    __shared__ float Lk[NB][NB + 1];
    __shared__ float inv[NB];
    const int z = blockIdx.y;
    const float *Lz = static_cast<const float *>(L.p[z]);
    float *Xz = static_cast<float *>(X.p[z]);
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
        const int i = idx / NB, j = idx % NB;
        Lk[i][j] = j <= i ? Lz[(size_t)(k0 + i) * D + k0 + j] : 0.f;
    }
    if (threadIdx.x < NB) inv[threadIdx.x] = 1.f / Lz[(size_t)(k0 + threadIdx.x) * D + k0 + threadIdx.x];
    __syncthreads();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= D) return;
    float x[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) x[j] = Xz[(size_t)(k0 + j) * D + c];
    if (!TRANS) {
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            x[j] *= inv[j];
#pragma unroll
            for (int i = j + 1; i < NB; ++i) x[i] -= Lk[i][j] * x[j];
        }
    } else {
#pragma unroll
        for (int j = NB - 1; j >= 0; --j) {
            x[j] *= inv[j];
#pragma unroll
            for (int i = 0; i < j; ++i) x[i] -= Lk[j][i] * x[j];
        }
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) Xz[(size_t)(k0 + j) * D + c] = x[j];
}

// partial[z][blockIdx.x] = sum over a strided share of i of X_z[i] * P_z[i] (double).
template <typename TX>
__global__ void __launch_bounds__(256) dot_partials_kernel(PtrBatch X, PtrBatch P, size_t n, double *partials) {
    const int z = blockIdx.y;
    const TX *Xz = static_cast<const TX *>(X.p[z]);
    const float *Pz = static_cast<const float *>(P.p[z]);
    double s = 0.0;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        s += (double)to_f32(Xz[i]) * (double)Pz[i];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    __shared__ double red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += red[w];
        partials[(size_t)z * gridDim.x + blockIdx.x] = t;
    }
}

// terms[k][z][p] for k = 0..4: tr(dW^T G dW), tr(dW^T C W), tr(W^T H W), tr(W^T G W), tr(W^T C W).
// One CTA of five warps per layer: warp k sums term k's partials (lane-strided, then a fixed
// shuffle tree), so the order of every sum is fixed.
__global__ void __launch_bounds__(160) finalize_eps_kernel(const double *terms, int nparts, int batch,
                                                            const int *status, float *eps, double *err_terms) {
    __shared__ double t[5];
    const int z = blockIdx.x, k = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const double *src = terms + ((size_t)k * batch + z) * nparts;
    double s = 0.0;
    for (int p = lane; p < nparts; p += 32) s += src[p];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    if (lane == 0) t[k] = s;
    __syncthreads();
    if (threadIdx.x != 0) return;
    const double E2 = t[0] - 2.0 * t[1] + t[2];
    const double T2 = t[3] + 2.0 * t[4] + t[2];
    float e = T2 == 0.0 ? 0.f : (float)(E2 / T2);
    if (status && status[z] != ISPA_OK) e = __int_as_float(0x7fc00000);
    eps[z] = e;
    if (err_terms) {
        err_terms[2 * z] = E2;
        err_terms[2 * z + 1] = T2;
    }
}

template <typename TW>
__global__ void add_delta_kernel(PtrBatch W, PtrBatch dW, PtrBatch out, size_t n) {
    const int z = blockIdx.y;
    const TW *Wz = static_cast<const TW *>(W.p[z]);
    const float *dz = static_cast<const float *>(dW.p[z]);
    TW *oz = static_cast<TW *>(out.p[z]);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        oz[i] = from_f32<TW>(to_f32(Wz[i]) + dz[i]);
}

__global__ void copy_f32_kernel(PtrBatch src, PtrBatch dst, size_t n) {
    const int z = blockIdx.y;
    const float4 *s = static_cast<const float4 *>(src.p[z]);
    float4 *d = static_cast<float4 *>(dst.p[z]);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x)
        d[i] = s[i];
}

}  // namespace

// ---- host side ----------------------------------------------------------------------

static GemmBatch make_gemm_batch(const PtrBatch &A, size_t offA, const PtrBatch &B, size_t offB, const PtrBatch &C,
                                 size_t offC, int batch, size_t eA, size_t eB) {
    GemmBatch g;
    for (int z = 0; z < batch; ++z) {
        g.A[z] = static_cast<const char *>(A.p[z]) + offA * eA;
        g.B[z] = static_cast<const char *>(B.p[z]) + offB * eB;
        g.C[z] = static_cast<char *>(C.p[z]) + offC * sizeof(float);
    }
    return g;
}

#define ISPA_TRY(x)                          \
    do {                                     \
        cudaError_t e_ = (x);                \
        if (e_ != cudaSuccess) return e_;    \
    } while (0)

// The five traces of the error and eps = E^2 / T^2 for dW given, Y = C W already in Y:
// t0 = tr(dW^T G dW), t1 = tr(dW^T Y), t2 = tr(W^T H W), t3 = tr(W^T G W), t4 = tr(W^T Y).
// On the tensor cores (tc) the quadratic forms are taken as dots with Gram matrices,
// tr(X^T S X) = sum_ij S_ij (X X^T)_ij: one symmetric product W W^T (its lower tiles only)
// dotted with G and H in its epilogue gives t3 and t2, dW dW^T dotted with G gives t0; t4 was
// taken when Y was formed and t1 too when t1_done (the solve's last product), which also left
// dW's split in (dw_hi, dw_lo) (else null: split here).
cudaError_t error_terms(const PtrBatch &G, const PtrBatch &H, const PtrBatch &W, ElemType wt, const PtrBatch &dW,
                        const PtrBatch &Y, const PtrBatch &P, float *Pc, float *split, double *terms, int nparts,
                        const int *status, float *eps, double *err_terms, int D, int batch, int *err_flag, bool tc,
                        bool t1_done, const float *dw_hi, const float *dw_lo, cudaStream_t s) {
    const size_t n = (size_t)D * D;
    const size_t ew = wt == ElemType::BF16 ? 2 : 4;
    const size_t bn = (size_t)batch * n;
    float *Ahi = split, *Alo = split + bn;
    const dim3 rgrid(nparts, batch);
    const bool wbf = wt == ElemType::BF16;
    double *t_dgd = terms, *t_dy = terms + (size_t)batch * nparts, *t_whw = terms + 2 * (size_t)batch * nparts,
           *t_wgw = terms + 3 * (size_t)batch * nparts;
    if (tc) {
        // W W^T (a bf16 W is exact in TF32: one term), dotted with G -> t3 and H -> t2
        ISPA_TRY(launch_split_tf32(W, wt, Ahi, wbf ? nullptr : Alo, D, D, false, batch, s));
        Tf32Opts ow;
        ow.sym = true;
        ow.dot_x = &G; ow.dot_out = t_wgw;
        ow.dot_x2 = &H; ow.dot_out2 = t_whw;
        ow.write_c = false;
        ISPA_TRY(launch_gemm_tf32x3(Ahi, wbf ? nullptr : Alo, Ahi, wbf ? nullptr : Alo, Pc, D, D, D, batch, err_flag,
                                    s, ow));
        // dW dW^T dotted with G -> t0 (dW split here unless its split is given)
        if (!dw_hi) {
            ISPA_TRY(launch_split_tf32(dW, ElemType::F32, Ahi, Alo, D, D, false, batch, s));
            dw_hi = Ahi;
            dw_lo = Alo;
        }
        Tf32Opts od;
        od.sym = true;
        od.dot_x = &G; od.dot_out = t_dgd;
        od.write_c = false;
        ISPA_TRY(launch_gemm_tf32x3(dw_hi, dw_lo, dw_hi, dw_lo, Pc, D, D, D, batch, err_flag, s, od));
        if (!t1_done) { dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(dW, Y, n, t_dy); note_launch(); }
    } else {
        GemmDesc full{D, D, D, D, D, D, true, false, ElemType::F32, ElemType::F32, ElemType::F32, 1.f, 0.f, false, batch};
        // t0 = tr(dW^T G dW)
        ISPA_TRY(launch_gemm_simt(full, make_gemm_batch(G, 0, dW, 0, P, 0, batch, 4, 4), s));
        dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(dW, P, n, t_dgd); note_launch();
        // t1 = tr(dW^T C W)
        dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(dW, Y, n, t_dy); note_launch();
        // t3 = tr(W^T G W), t2 = tr(W^T H W), t4 = tr(W^T C W)
        GemmDesc fw = full;
        fw.b_type = wt;
        ISPA_TRY(launch_gemm_simt(fw, make_gemm_batch(G, 0, W, 0, P, 0, batch, 4, ew), s));
        if (wbf) { dot_partials_kernel<bf16><<<rgrid, 256, 0, s>>>(W, P, n, t_wgw); note_launch(); }
        else { dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(W, P, n, t_wgw); note_launch(); }
        ISPA_TRY(launch_gemm_simt(fw, make_gemm_batch(H, 0, W, 0, P, 0, batch, 4, ew), s));
        if (wbf) { dot_partials_kernel<bf16><<<rgrid, 256, 0, s>>>(W, P, n, t_whw); note_launch(); }
        else { dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(W, P, n, t_whw); note_launch(); }
        double *t_wy = terms + 4 * (size_t)batch * nparts;
        if (wbf) { dot_partials_kernel<bf16><<<rgrid, 256, 0, s>>>(W, Y, n, t_wy); note_launch(); }
        else { dot_partials_kernel<float><<<rgrid, 256, 0, s>>>(W, Y, n, t_wy); note_launch(); }
    }
    ISPA_TRY(cudaGetLastError());
    finalize_eps_kernel<<<batch, 160, 0, s>>>(terms, nparts, batch, status, eps, err_terms); note_launch();
    ISPA_TRY(cudaGetLastError());

    return cudaSuccess;
}

// Y = C W for one batch of layers (W split into Whi/Wlo first when tc; then Y^T's split is left
// in the B_hi/B_lo blocks).
static cudaError_t c_times_w(const PtrBatch &C, const PtrBatch &W, ElemType wt, const PtrBatch &Y, float *Yc,
                             float *split, double *t_wy, int D, int batch, int *err_flag, bool tc, cudaStream_t s) {
    const size_t n = (size_t)D * D;
    const size_t ew = wt == ElemType::BF16 ? 2 : 4;
    const size_t bn = (size_t)batch * n;
    float *Ahi = split, *Alo = split + bn;
    float *Whi = split + 4 * bn, *Wlo = wt == ElemType::BF16 ? nullptr : split + 5 * bn;
    if (tc) {
        ISPA_TRY(launch_split_tf32(W, wt, Whi, Wlo, D, D, true, batch, s));
        ISPA_TRY(launch_split_tf32(C, ElemType::F32, Ahi, Alo, D, D, false, batch, s));
        // Y = C W, with t4 = tr(W^T Y) and Y's transposed split (the B operand of the solve's
        // first product) from the epilogue
        Tf32Opts o;
        o.dot_x = &W; o.dot_x_bf16 = wt == ElemType::BF16; o.dot_out = t_wy;
        o.split_hi = split + 2 * bn; o.split_lo = split + 3 * bn; o.split_t = true;
        ISPA_TRY(launch_gemm_tf32x3(Ahi, Alo, Whi, Wlo, Yc, D, D, D, batch, err_flag, s, o));
    } else {
        GemmDesc d{D, D, D, D, D, D, true, false, ElemType::F32, wt, ElemType::F32, 1.f, 0.f, false, batch};
        ISPA_TRY(launch_gemm_simt(d, make_gemm_batch(C, 0, W, 0, Y, 0, batch, 4, ew), s));
    }
    return cudaSuccess;
}

// The error of a given dW on given statistics (no solve): Y = C W, then the five traces.
// Scratch as for solve_batch (Y, P, the split blocks, terms).
cudaError_t error_batch(const PtrBatch &G, const PtrBatch &C, const PtrBatch &H, const PtrBatch &W, ElemType wt,
                        const PtrBatch &dW, const PtrBatch &Y, const PtrBatch &P, float *Yc, float *Pc, float *split,
                        double *terms, int nparts, float *eps, double *err_terms, int D, int batch, int *err_flag,
                        cudaStream_t s) {
    const bool tc = (D % 128 == 0) && split != nullptr;
    ISPA_TRY(c_times_w(C, W, wt, Y, Yc, split, terms + 4 * (size_t)batch * nparts, D, batch, err_flag, tc, s));
    return error_terms(G, H, W, wt, dW, Y, P, Pc, split, terms, nparts, nullptr, eps, err_terms, D, batch, err_flag,
                       tc, false, nullptr, nullptr, s);
}

// M = G + lambda I = L L^T and X = L^-1 into P, blocked by nb2 columns (512, 256 or 128): per
// block step k the cluster kernel factors and inverts the diagonal block (its
// inverse T_k is X's diagonal block), and the tensor cores (3xTF32) take the rest --
//   L_ik = A_ik T_k^T                    (the panel below, written to M with its split)
//   A_ij -= L_ik L_jk^T                  (the trailing update, lower tiles)
//   X_kc = T_k B_kc        (c < k)       (block row k of X from its accumulated right-hand side)
//   B_ic -= L_ik X_kc      (i > k, c <= k)
// with B = I at the start (P zeroed, the diagonal blocks set by the cluster kernel). Scratch: the
// split blocks 0, 1 (panel splits) and 4, 5 (T_k, B_k^T, X_k^T splits); blocks 2, 3 hold Y^T's
// split for the solve and are not touched. M and P hold `batch` contiguous D x D matrices.
static cudaError_t chol_inv_blocked(const PtrBatch &G, const PtrBatch &M, const PtrBatch &P, float *split, int D,
                                    float lambda, int batch, int *status, int *err_flag, int fill_blocks,
                                    cudaStream_t s) {
    // block width: 512 where it divides D (measured at D = 1,536: 6.8 ms against 6.9 for 384,
    // 7.0 for 256 and 768, 8.0 for 128), else 256, else 128; at most D / 2 (the scratch plan)
    const int nb2 = (D % 512 == 0 && D >= 1024) ? 512 : (D % 256 == 0 && D >= 768) ? 256 : 128;
    const int nblk = D / nb2;
    if (nblk == 1) return launch_chol_inv(G, M, P, D, lambda, batch, status, s);
    const size_t n = (size_t)D * D, bn = (size_t)batch * n;
    float *Mc = static_cast<float *>(M.p[0]), *Pc = static_cast<float *>(P.p[0]);
    // panel splits (block 0-1): A_ik then L_ik, each [batch][D - nb2][nb2]
    const size_t pan = (size_t)(D - nb2) * nb2;
    float *Ap_hi = split, *Ap_lo = Ap_hi + batch * pan, *Lp_hi = Ap_lo + batch * pan, *Lp_lo = Lp_hi + batch * pan;
    // blocks 4-5: T_k [batch][nb2][nb2], B_k^T [batch][D - nb2][nb2], X_k^T [batch][D][nb2]
    float *r45 = split + 4 * bn;
    const size_t tsz = (size_t)nb2 * nb2, xsz = (size_t)D * nb2;
    float *T_hi = r45, *T_lo = T_hi + batch * tsz, *Bt_hi = T_lo + batch * tsz, *Bt_lo = Bt_hi + batch * pan,
          *Xt_hi = Bt_lo + batch * pan, *Xt_lo = Xt_hi + batch * xsz;

    fill_shifted_kernel<<<dim3(fill_blocks, batch), 256, 0, s>>>(G, M, D, lambda); note_launch();
    ISPA_TRY(cudaGetLastError());
    ISPA_TRY(cudaMemsetAsync(Pc, 0, bn * sizeof(float), s));
    auto at = [&](const PtrBatch &X, size_t off) {
        PtrBatch o;
        for (int z = 0; z < batch; ++z) o.p[z] = static_cast<float *>(X.p[z]) + off;
        return o;
    };
    for (int k = 0; k < nblk; ++k) {
        const int r0 = k * nb2, rest = D - r0 - nb2;
        const size_t dk = (size_t)r0 * D + r0;
        ISPA_TRY(launch_chol_inv_block(at(M, dk), at(P, dk), nb2, D, batch, status, s));
        ISPA_TRY(launch_split_tf32(at(P, dk), ElemType::F32, T_hi, T_lo, nb2, nb2, false, batch, s, D));
        if (rest > 0) {
            const size_t below = (size_t)(r0 + nb2) * D + r0;
            ISPA_TRY(launch_split_tf32(at(M, below), ElemType::F32, Ap_hi, Ap_lo, rest, nb2, false, batch, s, D));
            Tf32Opts op;   // L_ik = A_ik T_k^T into M, and its split
            op.ldc = D; op.c_bstride = n;
            op.split_hi = Lp_hi; op.split_lo = Lp_lo;
            ISPA_TRY(launch_gemm_tf32x3(Ap_hi, Ap_lo, T_hi, T_lo, Mc + below, rest, nb2, nb2, batch, err_flag, s, op));
            Tf32Opts ou;   // A_ij -= L_ik L_jk^T, lower tiles
            ou.sym = true; ou.c_sub = true; ou.ldc = D; ou.c_bstride = n;
            ISPA_TRY(launch_gemm_tf32x3(Lp_hi, Lp_lo, Lp_hi, Lp_lo, Mc + below + nb2, rest, rest, nb2, batch, err_flag,
                                        s, ou));
        }
        // X_k^T's split holds r0 + nb2 rows per layer: X_kc^T (c < k) from the product, then T_k^T
        const size_t xt_bs = (size_t)(r0 + nb2) * nb2;
        if (k > 0) {
            ISPA_TRY(launch_split_tf32(at(P, (size_t)r0 * D), ElemType::F32, Bt_hi, Bt_lo, nb2, r0, true, batch, s, D));
            Tf32Opts ox;   // X_kc = T_k B_kc, T_k lower
            ox.a_tri = 1; ox.ldc = D; ox.c_bstride = n;
            ox.split_hi = Xt_hi; ox.split_lo = Xt_lo; ox.split_t = true; ox.split_bstride = xt_bs;
            ISPA_TRY(launch_gemm_tf32x3(T_hi, T_lo, Bt_hi, Bt_lo, Pc + (size_t)r0 * D, nb2, r0, nb2, batch, err_flag, s,
                                        ox));
        }
        if (rest > 0) {
            ISPA_TRY(launch_split_tf32(at(P, dk), ElemType::F32, Xt_hi + (size_t)r0 * nb2, Xt_lo + (size_t)r0 * nb2, nb2,
                                       nb2, true, batch, s, D, xt_bs));
            Tf32Opts ob;   // B_ic -= L_ik X_kc, c <= k
            ob.c_sub = true; ob.ldc = D; ob.c_bstride = n;
            ISPA_TRY(launch_gemm_tf32x3(Lp_hi, Lp_lo, Xt_hi, Xt_lo, Pc + (size_t)(r0 + nb2) * D, rest, r0 + nb2, nb2,
                                        batch, err_flag, s, ob));
        }
    }
    return cudaSuccess;
}

// Solve for one batch of layers. All pointers are device pointers, one per layer.
//   G, C, H: statistics; W: weights of type wt; dW: output (the batch's matrices contiguous,
//   dW.p[z] = dW.p[0] + z*D*D); M, Y: D*D float scratch each; P: D*D float scratch; Yc, Pc:
//   the Y and P blocks as contiguous batches; terms: 5 * batch * nparts doubles; status:
//   batch ints (zeroed).
cudaError_t solve_batch(const PtrBatch &G, const PtrBatch &C, const PtrBatch &H, const PtrBatch &W, ElemType wt,
                        const PtrBatch &dW, const PtrBatch &M, const PtrBatch &Y, const PtrBatch &P, float *Yc,
                        float *Pc, float *split, double *terms, int nparts, int *status, float *eps,
                        double *err_terms, const PtrBatch *w_new, int D, float lambda, int batch, int *err_flag,
                        cudaStream_t s) {
    const size_t n = (size_t)D * D;
    const int fill_blocks = (int)std::min<size_t>((n + 255) / 256, 1024);
    // D x D products on the tensor cores (3xTF32) when D is a multiple of 128; the split
    // operands live in `split`: A_hi, A_lo, B_hi, B_lo, W_hi, W_lo, each [batch][D][D].
    const bool tc = (D % 128 == 0) && split != nullptr;

    // Y = C W
    ISPA_TRY(c_times_w(C, W, wt, Y, Yc, split, terms + 4 * (size_t)batch * nparts, D, batch, err_flag, tc, s));

    const int nblk = D / NB;
    if (tc) {
        // M = G + lambda I = L L^T and X = L^-1 (in P)
        ISPA_TRY(chol_inv_blocked(G, M, P, split, D, lambda, batch, status, err_flag, fill_blocks, s));
        // Z = X Y, then dW = X^T Z (3xTF32; B operands are split transposed). Y^T's split is in the
        // B blocks (from Y's epilogue); Z leaves only its transposed split (in the W blocks, free
        // after Y), dW its own split (in the B blocks) for the error's dW dW^T.
        const size_t bn = (size_t)batch * n;
        float *Ahi = split, *Alo = split + bn, *Bhi = split + 2 * bn, *Blo = split + 3 * bn;
        float *Zhi = split + 4 * bn, *Zlo = split + 5 * bn;
        float *dWc = static_cast<float *>(dW.p[0]);
        ISPA_TRY(launch_split_tf32(P, ElemType::F32, Ahi, Alo, D, D, false, batch, s));
        Tf32Opts oz;
        oz.a_tri = 1;   // X lower
        oz.split_hi = Zhi; oz.split_lo = Zlo; oz.split_t = true;
        oz.write_c = false;
        ISPA_TRY(launch_gemm_tf32x3(Ahi, Alo, Bhi, Blo, dWc, D, D, D, batch, err_flag, s, oz));
        ISPA_TRY(launch_split_tf32(P, ElemType::F32, Ahi, Alo, D, D, true, batch, s));
        // X^T upper; t1 = tr(dW^T Y) from the epilogue
        Tf32Opts od;
        od.a_tri = 2;
        od.dot_x = &Y; od.dot_out = terms + (size_t)batch * nparts;
        od.split_hi = Bhi; od.split_lo = Blo;
        ISPA_TRY(launch_gemm_tf32x3(Ahi, Alo, Zhi, Zlo, dWc, D, D, D, batch, err_flag, s, od));
    } else {
        // M = G + lambda I, then the blocked Cholesky factorisation
        fill_shifted_kernel<<<dim3(fill_blocks, batch), 256, 0, s>>>(G, M, D, lambda); note_launch();
        ISPA_TRY(cudaGetLastError());
        for (int kb = 0; kb < nblk; ++kb) {
            const int k0 = kb * NB;
            potrf_diag_kernel<<<batch, NB, 0, s>>>(M, D, k0, status); note_launch();
            ISPA_TRY(cudaGetLastError());
            const int rest = D - k0 - NB;
            if (rest <= 0) break;
            trsm_panel_kernel<<<dim3((rest + NB - 1) / NB, batch), NB, 0, s>>>(M, D, k0); note_launch();
            ISPA_TRY(cudaGetLastError());
            GemmDesc d{rest, rest, NB, D, D, D, true, true, ElemType::F32, ElemType::F32, ElemType::F32, -1.f, 1.f,
                       true, batch};
            const size_t offA = (size_t)(k0 + NB) * D + k0;
            const size_t offC = (size_t)(k0 + NB) * D + k0 + NB;
            ISPA_TRY(launch_gemm_simt(d, make_gemm_batch(M, offA, M, offA, M, offC, batch, 4, 4), s));
        }
        // dW <- Y, solved in place: forward substitution L Z = Y, then backward L^T X = Z
        copy_f32_kernel<<<dim3(fill_blocks, batch), 256, 0, s>>>(Y, dW, n); note_launch();
        ISPA_TRY(cudaGetLastError());
        const dim3 tgrid((D + 127) / 128, batch);
        for (int kb = 0; kb < nblk; ++kb) {
            const int k0 = kb * NB;
            trsv_block_kernel<false><<<tgrid, 128, 0, s>>>(M, dW, D, k0); note_launch();
            ISPA_TRY(cudaGetLastError());
            const int rest = D - k0 - NB;
            if (rest <= 0) break;
            GemmDesc d{rest, D, NB, D, D, D, true, false, ElemType::F32, ElemType::F32, ElemType::F32, -1.f, 1.f,
                       false, batch};
            ISPA_TRY(launch_gemm_simt(
                d, make_gemm_batch(M, (size_t)(k0 + NB) * D + k0, dW, (size_t)k0 * D, dW, (size_t)(k0 + NB) * D, batch, 4, 4),
                s));
        }
        for (int kb = nblk - 1; kb >= 0; --kb) {
            const int k0 = kb * NB;
            trsv_block_kernel<true><<<tgrid, 128, 0, s>>>(M, dW, D, k0); note_launch();
            ISPA_TRY(cudaGetLastError());
            if (k0 == 0) break;
            // X[0:k0, :] -= (L[k0:k0+NB, 0:k0])^T X_k
            GemmDesc d{k0, D, NB, D, D, D, false, false, ElemType::F32, ElemType::F32, ElemType::F32, -1.f, 1.f, false,
                       batch};
            ISPA_TRY(launch_gemm_simt(d, make_gemm_batch(M, (size_t)k0 * D, dW, (size_t)k0 * D, dW, 0, batch, 4, 4), s));
        }
    }

    // Reconstruction error terms
    {
        const size_t bn = (size_t)batch * n;
        ISPA_TRY(error_terms(G, H, W, wt, dW, Y, P, Pc, split, terms, nparts, status, eps, err_terms, D, batch, err_flag,
                             tc, tc, tc ? split + 2 * bn : nullptr, tc ? split + 3 * bn : nullptr, s));
    }

    if (w_new) {
        if (wt == ElemType::BF16) { add_delta_kernel<bf16><<<dim3(fill_blocks, batch), 256, 0, s>>>(W, dW, *w_new, n); note_launch(); }
        else { add_delta_kernel<float><<<dim3(fill_blocks, batch), 256, 0, s>>>(W, dW, *w_new, n); note_launch(); }
        ISPA_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace ispa
