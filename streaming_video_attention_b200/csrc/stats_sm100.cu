// Ridge statistics from bf16 operands (placeholder routing to the CUDA-core GEMM until the
// tcgen05 GEMM lands).
#include "common.cuh"

namespace ispa {
cudaError_t launch_stats_bf16(const void *a_loc, const void *r, int n, int D, float *G, float *C, float *H,
                              int *err_flag, cudaStream_t s) {
    (void)err_flag;
    GemmDesc g{D, D, n, D, D, D, false, false, ElemType::BF16, ElemType::BF16, ElemType::F32, 1.f, 1.f, false, 1};
    GemmBatch b;
    b.A[0] = a_loc; b.B[0] = a_loc; b.C[0] = G;
    cudaError_t e = launch_gemm_simt(g, b, s);
    if (e != cudaSuccess) return e;
    b.A[0] = a_loc; b.B[0] = r; b.C[0] = C;
    e = launch_gemm_simt(g, b, s);
    if (e != cudaSuccess) return e;
    b.A[0] = r; b.B[0] = r; b.C[0] = H;
    return launch_gemm_simt(g, b, s);
}
}  // namespace ispa
