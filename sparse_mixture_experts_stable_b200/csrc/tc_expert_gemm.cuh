// Grouped bf16 tensor-core GEMM with weights on the M side (see tc_expert_gemm.cu).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "tc_gemm.cuh"

namespace moe {

struct TcxProblem {
    const void* w;             // bf16 weights (w_rows_total, K), row stride ldw: row g*w_rows_per_group + f
    const void* w2;            // second weight matrix for TC_EPI_SWIGLU (the up projection), else NULL
    int64_t ldw;
    int64_t w_rows_total;
    int64_t w_rows_per_group;
    const void* x;             // bf16 tokens (x_rows_total, K), row stride ldx: row g*x_rows_per_group + n
    int64_t ldx;
    int64_t x_rows_total;
    int64_t x_rows_per_group;
    int G;                     // groups (experts)
    int64_t features;          // output features per group
    int64_t max_tokens;        // token rows per group (C)
    int64_t K;
    const int32_t* rows;       // device (G) valid token rows per group, or NULL (= max_tokens)
    // Gathered token rows (TC_EPI_SWIGLU only): when non-NULL, token row n of group g
    // is row gather_index[g*max_tokens + n] of x (x_rows_total rows), read directly by
    // the kernel instead of from an expert-major copy; a negative index or n >= rows[g]
    // reads zeros.  x_rows_per_group is then unused.
    const int32_t* gather_index;
    void* out;                 // (G*out_rows_per_group, ldo): fp32 for TC_EPI_F32, else bf16
    int64_t ldo;
    int64_t out_rows_per_group;
    const void* bias;          // per feature: fp32 (TC_EPI_F32, shared by groups) or bf16 (+ g*bias_group_stride)
    int64_t bias_group_stride;
    int epilogue;              // TcEpilogue
    int32_t* status;
    // TC_EPI_SWIGLU: when non-NULL, the bf16 pre-activations are also stored, row for row
    // like out: a (gate) at column f, b (up) at column features + f, row stride ld_save.
    void* save_ab;
    int64_t ld_save;
    // tcw_gemm_run only: one device word of scratch for its tile counter (zeroed by the call, in stream order)
    uint32_t* tile_counter;
};

// Single-CTA kernel: 256 weight rows x up to 128 tokens per tile.
int tcx_gemm_run(const TcxProblem& p, cudaStream_t stream);

// SwiGLU gate/up (TC_EPI_SWIGLU) without gathered rows: 128 features (gate and
// up) x up to 256 tokens per tile, single-buffered TMEM (tc_wide_gemm.cu).
int tcw_gemm_run(const TcxProblem& p, cudaStream_t stream);


}  // namespace moe
