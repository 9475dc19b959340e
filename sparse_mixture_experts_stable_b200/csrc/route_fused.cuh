// The fused router (scores on tcgen05, softmax, stable top-k and gates in one
// kernel) used by moe_route for bf16 activations with E = 256 and k <= 8.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Whether the fused router handles this problem (bf16, K-major (E, D) weight).
bool route_fused_supported(int64_t T, int64_t D, int64_t ldx, const void* x, const void* w_ed, int32_t E,
                           int32_t k);

// CTAs the fused router launches for T tokens (= rows of its partial sums).
int route_fused_grid(int64_t T);

// Writes selected, gates, gates_f32 and (if given) the fp32 logits, and one row
// of per-expert counts and probability sums per CTA into part_counts /
// part_psum ((route_fused_grid(T), E) each).  Returns a moe_status.
int route_fused_run(const void* x, int64_t T, int64_t D, int64_t ldx, const void* w_ed, int32_t E,
                    const float* bias, int32_t k, float* logits_out, int64_t* selected, void* gates, int gates_bf16,
                    float* gates_f32, int32_t* part_counts, float* part_psum, int32_t* status, cudaStream_t stream);

}  // namespace moe
