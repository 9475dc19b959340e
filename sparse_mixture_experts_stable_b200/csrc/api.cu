// Small entry points: capacity, combine, weight transpose, status words, version.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "util_kernels.cuh"

namespace moe {

int device_sm_count() {
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 64) dev = 0;
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

}  // namespace moe

using namespace moe;

extern "C" const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported by this build";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_BAD_INDEX: return "expert index out of range";
        case MOE_ERR_NONFINITE: return "non-finite router logit";
        case MOE_ERR_TIMEOUT: return "device wait exceeded its time limit";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

extern "C" int moe_version(void) { return 100; }

extern "C" int moe_capacity(int64_t T, int32_t k, int32_t E, double capacity_factor, int64_t* C_out) {
    MOE_REQUIRE(C_out != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && k >= 1 && E >= 1 && k <= E, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(isfinite(capacity_factor) && capacity_factor > 0.0, MOE_ERR_INVALID_ARG);
    const double v = capacity_factor * (double)T * (double)k / (double)E;
    MOE_REQUIRE(v < 9.0e15, MOE_ERR_INVALID_ARG);
    int64_t c = (int64_t)ceil(v);
    *C_out = c < 1 ? 1 : c;
    return MOE_OK;
}

extern "C" int moe_combine(const void* ybuf, const int64_t* selected, const int64_t* slot, const void* gates,
                           moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C, int64_t N,
                           moe_base base_kind, const void* base, int64_t ldbase, void* y, int64_t ldy,
                           moe_dtype dtype, int32_t* dev_status, moe_stream_t stream) {
    MOE_REQUIRE(valid_dtype(dtype) && valid_dtype(gate_dtype), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(selected && slot && y && T >= 1 && k >= 1 && E >= 1 && C >= 0 && N >= 1 && ldy >= N,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(C == 0 || ybuf != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(base_kind == MOE_BASE_ZERO || base_kind == MOE_BASE_INPUT || base_kind == MOE_BASE_TENSOR,
                MOE_ERR_INVALID_ARG);
    const void* b = nullptr;
    if (base_kind != MOE_BASE_ZERO) {
        MOE_REQUIRE(base != nullptr && ldbase >= N, MOE_ERR_INVALID_ARG);
        b = base;
    }
    return combine_rows(ybuf, selected, slot, gates, gate_dtype, T, k, E, C, N, b, ldbase, y, ldy, dtype, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int moe_transpose_weights(const void* src, void* dst, int32_t E, int64_t K_in, int64_t N_out,
                                     moe_dtype dtype, moe_stream_t stream) {
    MOE_REQUIRE(valid_dtype(dtype) && src && dst && src != dst, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(E >= 1 && K_in >= 1 && N_out >= 1, MOE_ERR_INVALID_ARG);
    return transpose_matrices(src, dst, E, K_in, N_out, dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int moe_clear_status(int32_t* dev_status, moe_stream_t stream) {
    MOE_REQUIRE(dev_status != nullptr, MOE_ERR_INVALID_ARG);
    MOE_CUDA_TRY(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

extern "C" int moe_read_status(const int32_t* dev_status, moe_stream_t stream, int32_t* host_status) {
    MOE_REQUIRE(dev_status != nullptr && host_status != nullptr, MOE_ERR_INVALID_ARG);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    MOE_CUDA_TRY(cudaStreamSynchronize(s));
    MOE_CUDA_TRY(cudaMemcpy(host_status, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost));
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// moe_wait_probe: the library's bounded device wait, on a caller's flag
// ---------------------------------------------------------------------------
namespace moe {
namespace {

// One thread polls *flag (at most every microsecond) until it is non-zero or
// limit_ns has passed on the global timer; in the second case it records
// MOE_ERR_TIMEOUT and returns, as every wait inside the library does.
__global__ void wait_probe_kernel(const volatile uint32_t* flag, uint64_t limit_ns, int32_t* status) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    const uint64_t t0 = globaltimer_ns();
    while (*flag == 0u) {
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, MOE_ERR_TIMEOUT);
            return;
        }
        __nanosleep(1000);
    }
}

}  // namespace
}  // namespace moe

extern "C" int moe_wait_probe(const uint32_t* flag, int64_t limit_ns, int32_t* dev_status, moe_stream_t stream) {
    MOE_REQUIRE(flag && dev_status && limit_ns > 0 && (uint64_t)limit_ns <= kWaitLimitNs, MOE_ERR_INVALID_ARG);
    wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(flag, (uint64_t)limit_ns, dev_status);
    return launch_status();
}
