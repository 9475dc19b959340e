// moe_dispatch_static: moe_dispatch without a caller workspace.
//
// Some callers cannot allocate device memory: code that a host framework calls
// with nothing but input and output pointers (a plugin or custom-operator
// interface that owns the memory budget), where a cudaMalloc/cudaFree would
// synchronise the device and bypass that budget.  For them the slot scan's
// look-back state lives in a fixed, file-scope device array instead of a
// workspace.  The array is allocated by the CUDA runtime when the library's
// module is loaded on a device and stays there until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "dispatch_scan.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

// 4 MiB of look-back state: ceil(T / 128) * E + 1 words must fit.
constexpr size_t kStaticScanWords = size_t(1) << 20;
static __device__ __align__(256) uint32_t g_scan_scratch[kStaticScanWords];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_scan_scratch on the current device.  In host code the
// symbol name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, looked up once per device with that device current.
int scratch_address(void** out) {
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    MOE_REQUIRE(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED);
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        MOE_CUDA_TRY(cudaGetSymbolAddress(&p, g_scan_scratch));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_dispatch_static_max_state_bytes(void) { return kStaticScanWords * sizeof(uint32_t); }

extern "C" int moe_dispatch_static(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                                   const void* x, moe_dtype dtype, int64_t D, int64_t ldx, int64_t* slot,
                                   uint8_t* kept, int32_t* used, int32_t* overflow, int32_t* drops_per_token,
                                   int32_t* token_of_slot, void* xbuf, int32_t* dev_status, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = dispatch_check_args(selected, T, k, E, C, x, dtype, D, ldx, slot, kept, used, overflow, drops_per_token,
                                 token_of_slot, xbuf);
    if (rc != MOE_OK) return rc;
    if (dispatch_scan_state_bytes(T, E) > kStaticScanWords * sizeof(uint32_t)) return MOE_ERR_UNSUPPORTED;
    void* state = nullptr;
    rc = scratch_address(&state);
    if (rc != MOE_OK) return rc;
    // dispatch_scan_launch clears the state words it uses (stream-ordered) before the scan.
    rc = dispatch_scan_launch(selected, T, k, E, C, slot, kept, used, overflow, drops_per_token, token_of_slot,
                              state, dev_status, stream);
    if (rc != MOE_OK) return rc;
    if (x) rc = gather_rows(x, ldx, T, k, selected, slot, E, C, nullptr, xbuf, D, dtype, dev_status, stream);
    return rc;
}
