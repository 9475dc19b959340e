// fp32 grouped GEMM on the CUDA cores (FFMA), for the fp32 paths.
//
// C[g](m, n) = epilogue( sum_k A[g](m, k) * B[g](k, n) )
//   A(m, k) = a_trans ? A[k * lda + m] : A[m * lda + k]
//   B(k, n) = b_trans ? B[n * ldb + k] : B[k * ldb + n]
// Per group g the valid M (rows_mode 1) or K (rows_mode 2) can be limited by a
// device array rows[g]; rows outside the valid M are not written.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {

enum SimtEpilogue : int {
    SIMT_EPI_NONE = 0,
    SIMT_EPI_BIAS = 1,       // + bias[n]
    SIMT_EPI_BIAS_GELU = 2,  // gelu(acc + bias[n])
    SIMT_EPI_SILU_MUL = 3    // silu(acc) * C_old  (read-modify-write of C)
};

struct SimtGemm {
    const float* A = nullptr;
    int64_t lda = 0;
    bool a_trans = false;
    int64_t a_group_stride = 0;
    const float* B = nullptr;
    int64_t ldb = 0;
    bool b_trans = false;
    int64_t b_group_stride = 0;
    float* C = nullptr;
    int64_t ldc = 0;
    int64_t c_group_stride = 0;
    int64_t M = 0, N = 0, K = 0;
    int groups = 1;
    const int32_t* rows = nullptr;
    int rows_mode = 0;
    const float* bias = nullptr;
    int64_t bias_group_stride = 0;
    int epilogue = SIMT_EPI_NONE;
};

int simt_gemm_run(const SimtGemm& g, cudaStream_t stream);

}  // namespace moe
