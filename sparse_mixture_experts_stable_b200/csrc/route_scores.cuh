// Score helpers shared by the router kernels: an order-preserving integer key
// for fp32 scores (so that a top-k can compare integers and break ties by
// index) and the numerically stable sigmoid forms of the sigmoid scoring.
#pragma once

#include <math.h>
#include <stdint.h>

namespace moe {

// Order-preserving map from fp32 to uint32 (larger float -> larger key).  The
// score is canonicalised first so that -0 and +0 (equal as floats) share a key;
// NaN never reaches it (non-finite scores are replaced by -inf before).  Every
// key of a real score is above 0, so 0 serves as "no candidate yet".
__device__ __forceinline__ uint32_t order_key(float v) {
    if (v == 0.0f) v = 0.0f;
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inverse of order_key (-0 comes back as +0).
__device__ __forceinline__ float key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float sigmoid_stable_f(float z) {
    if (z >= 0.f) return 1.f / (1.f + expf(-z));
    const float ez = expf(z);
    return ez / (1.f + ez);
}

__device__ __forceinline__ float log_sigmoid_f(float z) {
    return z >= 0.f ? -log1pf(expf(-z)) : z - log1pf(expf(z));
}

}  // namespace moe
