// Row movement kernels shared by several entry points.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {

// Expert-major row buffers spread over ranks (expert parallelism): expert e
// lives on rank e / epr as local expert e % epr of that rank's (epr, C, .)
// buffer base[rank] (a peer buffer mapped into this process, or this rank's own).
constexpr int kMaxRanks = 64;
struct RankTable {
    void* base[kMaxRanks];
    int32_t ranks;
    int32_t epr;
    bool aligned16_all() const;
};

// dst[b] = src[b]^T for `batches` row-major (rows, cols) matrices -> (cols, rows).
int transpose_matrices(const void* src, void* dst, int64_t batches, int64_t rows, int64_t cols, moe_dtype dtype,
                       cudaStream_t stream);

// Token-major scatter into an expert-major buffer: for every kept assignment
// (slot[t,j] >= 0) copy src row t (times scale[t,j] if scale != NULL, in fp32)
// into dst[(selected[t,j] * C + slot[t,j]) * D ...].  Each src row is read once.
// With tab != NULL the rows go to the rank buffers of tab instead (dst unused).
int gather_rows(const void* src, int64_t lds, int64_t T, int32_t k, const int64_t* selected, const int64_t* slot,
                int32_t E, int64_t C, const float* scale, void* dst, int64_t D, moe_dtype dtype,
                int32_t* status, cudaStream_t stream, const RankTable* tab = nullptr);

// y[t] = base[t] + sum_{j asc, slot >= 0} gate[t,j] * ybuf[selected[t,j], slot[t,j]]
// (gate = 1 when gates == NULL; base absent when base == NULL).  With
// tab != NULL the rows are read from the rank buffers of tab (ybuf unused).
int combine_rows(const void* ybuf, const int64_t* selected, const int64_t* slot, const void* gates,
                 moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C, int64_t N, const void* base,
                 int64_t ldbase, void* y, int64_t ldy, moe_dtype dtype, int32_t* status, cudaStream_t stream,
                 const RankTable* tab = nullptr);

}  // namespace moe
