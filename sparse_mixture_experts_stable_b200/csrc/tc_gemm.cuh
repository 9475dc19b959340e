// Grouped bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// out[g, m, n] = epilogue( sum_k A[g, m, k] * B[g, n, k] )     for m < rows[g]
//
// Both operands are K-major bf16 (A: activations (rows, K); B: weights in the
// (out, in) layout), or B is MN-major (b_mn_major: B stored (K, N), N
// contiguous, e.g. a weight read transposed), fp32 accumulation in tensor memory.  One persistent CTA per
// SM walks a static list of (group, m-tile, n-tile) tiles whose length depends on
// the per-group row counts read on the device.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

enum TcEpilogue : int {
    TC_EPI_F32 = 0,        // fp32 out (+ optional fp32 column bias)      -- router scores
    TC_EPI_BF16 = 1,       // bf16 out                                    -- linear / down
    TC_EPI_BF16_BIAS = 2,  // bf16 out, + bf16 bias                       -- GELU MLP fc2
    TC_EPI_GELU_BIAS = 3,  // bf16 gelu(acc + bias)                       -- GELU MLP fc1
    TC_EPI_SWIGLU = 4,     // dual B: bf16 silu(acc_gate) * acc_up        -- SwiGLU gate/up
    TC_EPI_F32_DUAL = 5,   // dual B: fp32 acc_gate -> out[., n], acc_up -> out[., N + n]   -- [a | b] recompute
    TC_EPI_SWIGLU_BWD = 6  // acc = dh; with [a | b] = ab (bf16, rows of out): h = silu(a) b -> h,
                           // [dh b silu'(a) | dh silu(a)] -> out (bf16, 2N wide)  -- SwiGLU backward
};

struct TcGemmProblem {
    const void* a;            // bf16, row-major (a_rows_total, K), row stride lda
    int64_t lda;
    int64_t a_rows_total;
    int64_t a_rows_per_group; // row offset of group g in A
    const void* b;            // bf16 (b_rows_total, K), row stride ldb
    const void* b2;           // second B for TC_EPI_SWIGLU (same shape), else NULL; with b_mn_major
                              // and k_split > 0: the rows of K positions >= k_split (row k - k_split)
    int64_t ldb;
    int64_t b_rows_total;
    int64_t b_rows_per_group; // row offset of group g in B (b_mn_major: K rows per group)
    bool b_mn_major;          // B(k, n) = b[(g * b_rows_per_group + k) * ldb + n]; epilogues F32 / BF16 only,
                              // UMMA N a multiple of 64, k_split a multiple of 64
    int64_t k_split;
    bool a_mn_major;          // A(m, k) = a[(g * a_rows_per_group + k) * lda + m] (with b_mn_major, F32 out):
                              // both operands hold K on their rows; with k_rows the rows of a group's last
                              // K block past k_rows[g] are cleared in shared memory before the MMAs
    int G;                    // groups
    int64_t M;                // max rows per group
    int64_t N;                // output columns per group
    int64_t K;
    const int32_t* rows;      // device (G) valid rows per group, or NULL (= M)
    const int32_t* k_rows;    // device (G) valid K per group (operands zero past it), or NULL (= K)
    void* out;                // fp32 or bf16 per epilogue
    int64_t ldo;
    int64_t out_rows_per_group;
    void* out2;               // with a_mn_major and m_split > 0: rows m >= m_split of each group go to
    int64_t m_split;          // out2 (row m - m_split, same ldo and out_rows_per_group); a multiple of 128
    const void* ab;           // TC_EPI_SWIGLU_BWD: bf16 [a | b] with the rows and row stride of out
    void* h;                  // TC_EPI_SWIGLU_BWD: bf16 h = silu(a) b, row stride N
    const void* bias;         // fp32 (TC_EPI_F32) or bf16, per output column
    int64_t bias_group_stride;
    int epilogue;
    int32_t* status;
};

// Validates alignment, encodes the tensor maps and launches.  Returns a moe_status.
int tc_gemm_run(const TcGemmProblem& p, cudaStream_t stream);

// 2-D bf16 TMA map over a (rows, inner) row-major matrix with row stride
// ld_elems: box = box_rows x 64 elements, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows);

// The same for fp32 elements: box = box_rows x 32 elements (128 bytes).
bool make_map_f32(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows);
// fp32, box_rows x 32, 128-byte swizzle of 32-byte chunks: MN-major tf32 operands.
bool make_map_f32_mn(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows);

}  // namespace moe
