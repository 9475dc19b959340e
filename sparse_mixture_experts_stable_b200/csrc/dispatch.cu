// moe_dispatch: greedy position-priority slots as a single-pass per-expert
// prefix count (decoupled look-back), then the row gather into (E, C, D).
//
// The assignment stream is ordered by (token asc, route slot asc).  Each block
// owns kScanTokens consecutive tokens.  Inside a block, warps own consecutive
// 32-element chunks; __match_any_sync groups equal experts in a chunk, so a rank
// is (block prefix) + (earlier warps) + (earlier chunks) + (earlier lanes).
// Blocks take their position from an atomic ticket, so a block only ever waits
// for blocks that are already running; each wait is bounded in time.
#include <cuda_runtime.h>

#include "common.cuh"
#include "dispatch_scan.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanTokens = 128;  // 128 blocks at T = 16384: most SMs take part
constexpr uint32_t kFlagAgg = 1u << 30;   // block aggregate published
constexpr uint32_t kFlagPre = 2u << 30;   // inclusive prefix published
constexpr uint32_t kValMask = (1u << 30) - 1;

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

constexpr int kBatch = 8;  // chunk keys fetched together per warp

// Expert index of stream element li of this block, or -1 when the element does
// not exist or (reported to status when given) lies outside [0, E).
__device__ __forceinline__ int load_key(const int64_t* __restrict__ selected, int64_t base_i, int n_el, int li,
                                        bool chunk_ok, int E, int32_t* status) {
    if (!chunk_ok || li >= n_el) return -1;
    const int64_t e = selected[base_i + li];
    if (e >= 0 && e < E) return (int)e;
    if (status) set_status(status, MOE_ERR_BAD_INDEX);
    return -1;
}

__global__ void __launch_bounds__(kScanThreads)
    slot_scan_kernel(const int64_t* __restrict__ selected, int64_t T, int k, int E, int64_t C, int nblocks,
                     int64_t* __restrict__ slot, uint8_t* __restrict__ kept, int32_t* __restrict__ used,
                     int32_t* __restrict__ overflow, int32_t* __restrict__ drops,
                     int32_t* __restrict__ token_of_slot, uint32_t* __restrict__ state, uint32_t* ticket,
                     int32_t* status, const int32_t* __restrict__ rank_base, int64_t token_base) {
    extern __shared__ int s_dyn[];
    int* s_off = s_dyn;                          // [kScanWarps][E]: per-warp running rank
    int* s_drop = s_off + kScanWarps * E;        // [kScanTokens]
    __shared__ int s_bid;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_bid = (int)atomicAdd(ticket, 1u);
    for (int i = threadIdx.x; i < kScanWarps * E; i += kScanThreads) s_off[i] = 0;
    for (int i = threadIdx.x; i < kScanTokens; i += kScanThreads) s_drop[i] = 0;
    __syncthreads();
    const int bid = s_bid;

    const int64_t t0 = (int64_t)bid * kScanTokens;
    const int64_t ntok = (T - t0) < kScanTokens ? (T - t0) : kScanTokens;
    const int64_t base_i = t0 * k;
    const int n_el = (int)(ntok * k);
    const int nchunks = (n_el + 31) / 32;
    const int cpw = (nchunks + kScanWarps - 1) / kScanWarps;
    const int c_begin = warp * cpw;
    const int c_end = (c_begin + cpw) < nchunks ? (c_begin + cpw) : nchunks;
    int* my_off = s_off + warp * E;

    // pass 1: per-warp histogram of the warp's chunks (keys fetched kBatch chunks at a time)
    for (int c0 = c_begin; c0 < c_end; c0 += kBatch) {
        int keys[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) keys[u] = load_key(selected, base_i, n_el, (c0 + u) * 32 + lane, c0 + u < c_end, E,
                                                          status);
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (c0 + u >= c_end) break;
            const int key = keys[u];
            const uint32_t match = __match_any_sync(0xffffffffu, key);
            if (key >= 0 && (__ffs(match) - 1) == lane) my_off[key] += __popc(match);
        }
    }
    __syncthreads();

    // per expert: warp offsets, block aggregate, look-back for the block prefix
    for (int e = threadIdx.x; e < E; e += kScanThreads) {
        int run = 0;
        for (int w = 0; w < kScanWarps; ++w) {
            const int v = s_off[w * E + e];
            s_off[w * E + e] = run;
            run += v;
        }
        const uint32_t agg = (uint32_t)run;
        uint32_t* mine = state + (int64_t)bid * E + e;
        uint32_t excl = 0;
        if (bid == 0) {
            st_release(mine, kFlagPre | agg);
        } else {
            st_release(mine, kFlagAgg | agg);
            int p = bid - 1;
            uint64_t t_start = 0;
            bool timed_out = false;
            while (p >= 0) {
                const uint32_t w = ld_acquire(state + (int64_t)p * E + e);
                const uint32_t flag = w & ~kValMask;
                if (flag == 0) {
                    const uint64_t now = globaltimer_ns();
                    if (t_start == 0) t_start = now;
                    else if (now - t_start > kWaitLimitNs) {
                        timed_out = true;
                        break;
                    }
                    continue;
                }
                excl += w & kValMask;
                if (flag == kFlagPre) break;
                --p;
            }
            if (timed_out) set_status(status, MOE_ERR_TIMEOUT);
            st_release(mine, kFlagPre | ((excl + agg) & kValMask));
        }
        // expert parallelism: the assignments of lower ranks come first
        const int rb = rank_base ? rank_base[e] : 0;
        for (int w = 0; w < kScanWarps; ++w) s_off[w * E + e] += (int)excl + rb;
        if (bid == nblocks - 1 && rank_base == nullptr) {
            const int64_t total = (int64_t)excl + agg;
            const int64_t u = total < C ? total : C;
            used[e] = (int32_t)u;
            overflow[e] = (int32_t)(total - u);
        }
    }
    __syncthreads();

    // pass 2: ranks -> slots
    for (int c0 = c_begin; c0 < c_end; c0 += kBatch) {
      int keys[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
          keys[u] = load_key(selected, base_i, n_el, (c0 + u) * 32 + lane, c0 + u < c_end, E, nullptr);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + u;
        if (c >= c_end) break;
        const int li = c * 32 + lane;
        const int key = keys[u];
        const uint32_t match = __match_any_sync(0xffffffffu, key);
        int rank = 0;
        if (key >= 0) rank = my_off[key] + __popc(match & lanemask_lt());
        __syncwarp();
        if (key >= 0 && (__ffs(match) - 1) == lane) my_off[key] += __popc(match);
        __syncwarp();
        if (li < n_el) {
            const int64_t i = base_i + li;
            const int64_t t = i / k;
            if (key >= 0 && rank < C) {
                slot[i] = rank;
                kept[i] = 1;
                if (token_of_slot) token_of_slot[(int64_t)key * C + rank] = (int32_t)(token_base + t);
            } else {
                slot[i] = -1;
                kept[i] = 0;
                atomicAdd(&s_drop[t - t0], 1);
            }
        }
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ntok; i += kScanThreads) drops[t0 + i] = s_drop[i];
}

}  // namespace

size_t dispatch_scan_state_bytes(int64_t T, int32_t E) {
    const int64_t nb = (T + kScanTokens - 1) / kScanTokens;
    return align_up((size_t)nb * E * sizeof(uint32_t) + sizeof(uint32_t), 256);
}

int dispatch_scan_launch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C, int64_t* slot,
                         uint8_t* kept, int32_t* used, int32_t* overflow, int32_t* drops, int32_t* token_of_slot,
                         void* state_mem, int32_t* status, cudaStream_t stream, const int32_t* rank_base,
                         int64_t token_base) {
    const int64_t nb = (T + kScanTokens - 1) / kScanTokens;
    uint32_t* state = static_cast<uint32_t*>(state_mem);
    uint32_t* ticket = state + nb * E;
    MOE_CUDA_TRY(cudaMemsetAsync(state, 0, (size_t)nb * E * sizeof(uint32_t) + sizeof(uint32_t), stream));
    if (C > 0 && token_of_slot)
        MOE_CUDA_TRY(cudaMemsetAsync(token_of_slot, 0xFF, (size_t)E * C * sizeof(int32_t), stream));
    const size_t smem = sizeof(int) * ((size_t)kScanWarps * E + kScanTokens);
    if (smem > 48 * 1024)
        MOE_CUDA_TRY(cudaFuncSetAttribute(slot_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    slot_scan_kernel<<<(unsigned)nb, kScanThreads, smem, stream>>>(selected, T, k, E, C, (int)nb, slot, kept, used,
                                                                   overflow, drops, token_of_slot, state, ticket,
                                                                   status, rank_base, token_base);
    return launch_status();
}

int dispatch_check_args(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C, const void* x,
                        moe_dtype dtype, int64_t D, int64_t ldx, const int64_t* slot, const uint8_t* kept,
                        const int32_t* used, const int32_t* overflow, const int32_t* drops,
                        const int32_t* token_of_slot, const void* xbuf) {
    MOE_REQUIRE(selected && slot && kept && used && overflow && drops, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(C == 0 || token_of_slot != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && k >= 1 && E >= 1 && C >= 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T * (int64_t)k < (int64_t(1) << 30) && C < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(E <= 2048 && k <= 64, MOE_ERR_UNSUPPORTED);  // scan smem: (16 E + 128) * 4 bytes
    if (x) {
        MOE_REQUIRE(valid_dtype(dtype) && (xbuf || C == 0) && D >= 1 && ldx >= D, MOE_ERR_INVALID_ARG);
    }
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_dispatch_workspace_size(int64_t T, int32_t k, int32_t E) {
    (void)k;
    if (T < 1 || E < 1) return 0;
    return dispatch_scan_state_bytes(T, E);
}

extern "C" int moe_dispatch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C, const void* x,
                            moe_dtype dtype, int64_t D, int64_t ldx, int64_t* slot, uint8_t* kept, int32_t* used,
                            int32_t* overflow, int32_t* drops_per_token, int32_t* token_of_slot, void* xbuf,
                            int32_t* dev_status, void* workspace, size_t workspace_bytes, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = dispatch_check_args(selected, T, k, E, C, x, dtype, D, ldx, slot, kept, used, overflow, drops_per_token,
                                 token_of_slot, xbuf);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(workspace != nullptr && workspace_bytes >= dispatch_scan_state_bytes(T, E), MOE_ERR_WORKSPACE);
    rc = dispatch_scan_launch(selected, T, k, E, C, slot, kept, used, overflow, drops_per_token, token_of_slot,
                              workspace, dev_status, stream);
    if (rc != MOE_OK) return rc;
    if (x) rc = gather_rows(x, ldx, T, k, selected, slot, E, C, nullptr, xbuf, D, dtype, dev_status, stream);
    return rc;
}
