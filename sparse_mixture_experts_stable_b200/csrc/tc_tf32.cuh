// fp32 grouped GEMM on the tcgen05 tensor cores with split-tf32 operands.
//
// Operand forms, row limits and epilogues of F32Gemm (f32_gemm.cuh):
//   C[g](m, n) = epilogue( sum_k A[g](m, k) * B[g](k, n) )
// Every fp32 operand x is split into hi = x rounded to tf32 (10 mantissa bits)
// and lo = x - hi (exact in fp32), and the product is taken as
//   a_hi*b_hi + a_hi*b_lo + a_lo*b_hi
// in fp32 accumulation (three tf32 MMAs per K step; the dropped a_lo*b_lo is
// below 2^-21 of |a*b|), which keeps the result at fp32 accuracy.  The split
// operands are written K-major into a caller workspace first.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "f32_gemm.cuh"

namespace moe {

// Workspace bytes tf32x3_gemm_run needs for this problem.
size_t tf32x3_workspace_size(const F32Gemm& g);

// Runs the problem; returns a moe_status (MOE_ERR_WORKSPACE if the workspace is short).
int tf32x3_gemm_run(const F32Gemm& g, void* workspace, size_t workspace_bytes, int32_t* status,
                    cudaStream_t stream);

}  // namespace moe
