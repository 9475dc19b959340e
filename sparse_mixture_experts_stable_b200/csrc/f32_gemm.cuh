// Problem form of the fp32 grouped GEMMs (run on the tensor cores as
// split-tf32 products by tf32x3_gemm_run, tc_tf32.cuh).
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

enum F32Epilogue : int {
    F32_EPI_NONE = 0,
    F32_EPI_BIAS = 1,       // + bias[n]
    F32_EPI_BIAS_GELU = 2,  // gelu(acc + bias[n])
    F32_EPI_SILU_MUL = 3    // silu(acc) * C_old  (read-modify-write of C)
};

struct F32Gemm {
    // A and B are fp32, or bf16 when a_bf16 / b_bf16 is set (read through the
    // same pointers; products still in fp32 accuracy).
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
    int epilogue = F32_EPI_NONE;
    bool a_bf16 = false;
    bool b_bf16 = false;
};

}  // namespace moe
