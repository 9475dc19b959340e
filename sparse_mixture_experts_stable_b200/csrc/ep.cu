// Expert parallelism: R ranks, one GPU each, every rank holding T_r tokens and
// E / R experts (rank r owns experts [r E/R, (r+1) E/R)).
//
// Capacity semantics: the layer over the R ranks is the layer over the whole
// batch, tokens ordered rank-major.  Expert e keeps at most
// C = ceil(cf * T * k / E) assignments in that global order; with T and E both
// split R ways the formula gives the same C as on one GPU (the numpy-layer
// page, section 1 item 2), and the greedy position priority becomes: rank r's
// assignments to e start at slot sum_{r' < r} count_{r'}[e].  The slot of every
// assignment is therefore known on its own rank after one exchange of the E
// pre-drop counts per rank, and the rows move in a single pass:
//   moe_ep_plan      per-expert slot base for this rank, global used/overflow
//   moe_ep_dispatch  slot scan from that base, then the row gather writing
//                    each kept row straight into the owner rank's expert-major
//                    buffer (peer memory mapped into this process)
//   moe_ep_combine   the gate-weighted combine reading each kept row from the
//                    owner rank's output buffer (peer memory)
// The exchange of A*D rows each way that the Module 7 page sizes for expert
// parallelism is thus done by the gather and combine kernels themselves over
// NVLink, with no staging copy.  Between the calls the ranks synchronise (the
// counts exchange and two barriers per step, issued by the caller).
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "dispatch_scan.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

// rank_base[e] = sum_{r < rank} counts_all[r][e];  total = sum_r counts_all[r][e]
// used = min(total, C), overflow = total - used (totals saturate at INT32_MAX).
__global__ void ep_plan_kernel(const int32_t* __restrict__ counts_all, int R, int rank, int E, int64_t C,
                               int32_t* __restrict__ rank_base, int32_t* __restrict__ used,
                               int32_t* __restrict__ overflow, int32_t* __restrict__ counts_total) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        int64_t pre = 0, tot = 0;
        for (int r = 0; r < R; ++r) {
            const int64_t c = counts_all[(int64_t)r * E + e];
            if (r < rank) pre += c;
            tot += c;
        }
        const int64_t lim = 0x7fffffff;
        pre = pre < lim ? pre : lim;
        tot = tot < lim ? tot : lim;
        const int64_t u = tot < C ? tot : C;
        rank_base[e] = (int32_t)pre;
        if (used) used[e] = (int32_t)u;
        if (overflow) overflow[e] = (int32_t)(tot - u);
        if (counts_total) counts_total[e] = (int32_t)tot;
    }
}

int fill_table(RankTable& t, const void* const* ptrs, int32_t R, int32_t E) {
    MOE_REQUIRE(ptrs != nullptr, MOE_ERR_INVALID_ARG);
    memset(&t, 0, sizeof(t));
    for (int r = 0; r < R; ++r) {
        MOE_REQUIRE(ptrs[r] != nullptr, MOE_ERR_INVALID_ARG);
        t.base[r] = const_cast<void*>(ptrs[r]);
    }
    t.ranks = R;
    t.epr = E / R;
    return MOE_OK;
}

// A failed runtime call also leaves its code in the per-thread last-error slot;
// clear it so that a later launch check does not report it again.
#define EP_CUDA_TRY(expr)                  \
    do {                                   \
        if ((expr) != cudaSuccess) {       \
            (void)cudaGetLastError();      \
            return MOE_ERR_CUDA;           \
        }                                  \
    } while (0)

using GetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetAddressRangeFn address_range_fn() {
    static GetAddressRangeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetAddressRangeFn>(ptr);
    });
    return fn;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_ep_plan(const int32_t* counts_all, int32_t R, int32_t rank, int32_t E, int64_t C,
                           int32_t* rank_base, int32_t* used, int32_t* overflow, int32_t* counts_total,
                           moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(counts_all && rank_base, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(R >= 1 && rank >= 0 && rank < R && E >= 1 && C >= 0, MOE_ERR_INVALID_ARG);
    const int threads = 256;
    const unsigned blocks = (unsigned)((E + threads - 1) / threads);
    ep_plan_kernel<<<blocks, threads, 0, stream>>>(counts_all, R, rank, E, C, rank_base, used, overflow,
                                                   counts_total);
    return launch_status();
}

extern "C" int moe_ep_dispatch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                               const int32_t* rank_base, int64_t token_base, const void* x, moe_dtype dtype,
                               int64_t D, int64_t ldx, void* const* xbuf_ranks, int32_t R, int64_t* slot,
                               uint8_t* kept, int32_t* drops_per_token, int32_t* token_of_slot, int32_t* dev_status,
                               void* workspace, size_t workspace_bytes, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(selected && rank_base && slot && kept && drops_per_token, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && k >= 1 && E >= 1 && C >= 0 && token_base >= 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(R >= 1 && E % R == 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(R <= kMaxRanks, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(T * (int64_t)k < (int64_t(1) << 30) && C < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(token_base + T < (int64_t(1) << 31), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(E <= 2048 && k <= 64, MOE_ERR_UNSUPPORTED);
    RankTable tab;
    if (x) {
        MOE_REQUIRE(valid_dtype(dtype) && D >= 1 && ldx >= D, MOE_ERR_INVALID_ARG);
        if (C > 0) {
            const int rc = fill_table(tab, xbuf_ranks, R, E);
            if (rc != MOE_OK) return rc;
        }
    }
    MOE_REQUIRE(workspace != nullptr && workspace_bytes >= dispatch_scan_state_bytes(T, E), MOE_ERR_WORKSPACE);
    int rc = dispatch_scan_launch(selected, T, k, E, C, slot, kept, nullptr, nullptr, drops_per_token, token_of_slot,
                                  workspace, dev_status, stream, rank_base, token_base);
    if (rc != MOE_OK) return rc;
    if (x && C > 0)
        rc = gather_rows(x, ldx, T, k, selected, slot, E, C, nullptr, nullptr, D, dtype, dev_status, stream, &tab);
    return rc;
}

extern "C" int moe_ep_combine(const void* const* ybuf_ranks, int32_t R, const int64_t* selected, const int64_t* slot,
                              const void* gates, moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C,
                              int64_t N, moe_base base_kind, const void* base, int64_t ldbase, void* y, int64_t ldy,
                              moe_dtype dtype, int32_t* dev_status, moe_stream_t stream) {
    MOE_REQUIRE(valid_dtype(dtype) && valid_dtype(gate_dtype), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(selected && slot && y && T >= 1 && k >= 1 && E >= 1 && C >= 0 && N >= 1 && ldy >= N,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(R >= 1 && E % R == 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(R <= kMaxRanks, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(base_kind == MOE_BASE_ZERO || base_kind == MOE_BASE_INPUT || base_kind == MOE_BASE_TENSOR,
                MOE_ERR_INVALID_ARG);
    const void* b = nullptr;
    if (base_kind != MOE_BASE_ZERO) {
        MOE_REQUIRE(base != nullptr && ldbase >= N, MOE_ERR_INVALID_ARG);
        b = base;
    }
    RankTable tab;
    if (C > 0) {
        const int rc = fill_table(tab, ybuf_ranks, R, E);
        if (rc != MOE_OK) return rc;
    } else {
        memset(&tab, 0, sizeof(tab));
        tab.ranks = 0;
        tab.epr = E / R;
    }
    return combine_rows(nullptr, selected, slot, gates, gate_dtype, T, k, E, C, N, b, ldbase, y, ldy, dtype,
                        dev_status, reinterpret_cast<cudaStream_t>(stream), &tab);
}

extern "C" int moe_ipc_export(const void* dev_ptr, void* handle, int64_t* offset) {
    MOE_REQUIRE(dev_ptr && handle && offset, MOE_ERR_INVALID_ARG);
    GetAddressRangeFn fn = address_range_fn();
    MOE_REQUIRE(fn != nullptr, MOE_ERR_CUDA);
    CUdeviceptr base = 0;
    size_t size = 0;
    MOE_REQUIRE(fn(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) == CUDA_SUCCESS, MOE_ERR_CUDA);
    cudaIpcMemHandle_t h;
    EP_CUDA_TRY(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)));
    static_assert(sizeof(h) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    memcpy(handle, &h, sizeof(h));
    *offset = (int64_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
    return MOE_OK;
}

extern "C" int moe_ipc_import(const void* handle, void** mapping) {
    MOE_REQUIRE(handle && mapping, MOE_ERR_INVALID_ARG);
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof(h));
    EP_CUDA_TRY(cudaIpcOpenMemHandle(mapping, h, cudaIpcMemLazyEnablePeerAccess));
    return MOE_OK;
}

extern "C" int moe_ipc_close(void* mapping) {
    MOE_REQUIRE(mapping != nullptr, MOE_ERR_INVALID_ARG);
    EP_CUDA_TRY(cudaIpcCloseMemHandle(mapping));
    return MOE_OK;
}
