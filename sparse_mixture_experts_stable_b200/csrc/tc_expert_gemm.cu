// Grouped bf16 GEMM with the weights on the MMA's M side ("features x tokens"),
// for the expert FFNs and the router on sm_100a.
//
//   out[g, n, f] = epilogue( sum_k W[g, f, k] * X[g, n, k] )      n < rows[g]
//
// A tile is 256 weight rows x n_cur tokens: two M=128 MMAs (weight rows f..f+127
// and f+128..f+255, or for SwiGLU the gate and the up rows of features
// f..f+127) share one token tile and accumulate into two 128-column TMEM
// ranges.  n_cur is the group's remaining token count rounded up to 16 (at most
// 128), set per tile in the instruction descriptor, so a ragged expert wastes at
// most 15 token rows.  With few tokens per expert and many features, a
// wide-feature, short-token tile also re-reads the least data: the token tile is
// loaded once per 256 weight rows.  For SwiGLU every thread holds gate and up of
// the same feature and emits silu(g)*u directly.
//
// Warp roles (192 threads, one persistent CTA per SM): warp 0 issues TMA loads
// into a 4-stage ring, warp 1 owns TMEM (2 x 256 columns, double-buffered) and
// issues tcgen05.mma, warps 2..5 drain the accumulator.  The epilogue holds one
// feature per thread and 32 tokens per TMEM load; for each token the 32 lanes
// of a warp store 32 consecutive features of that token's row, so every store
// instruction writes one contiguous run.  All mbarrier waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_expert_gemm.cuh"
#include "tc_gemm.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kM = 128;       // features per tile (UMMA M)
constexpr int kBK = 64;       // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kGatherThreads = 128;  // gathered token rows: four more warps fill the token tile
constexpr int kGatherLag = 2;       // stages a gather thread keeps in flight before signalling
constexpr int kMaxGroups = 1024;
constexpr int kStageBytes = 48 * 1024;  // two weight tiles (2 x 16 KB) + 128 token rows (16 KB)
constexpr int kNT = 128;                // token rows per tile (TMA box height)
constexpr int kAccCols = 256;           // TMEM columns per accumulator buffer
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

struct XParams {
    int G;
    int64_t w_rows_per_group;
    int64_t x_rows_per_group;
    int64_t features;
    int64_t max_tokens;
    int f_tiles;
    int feat_per_tile;  // 128 (SwiGLU: gate and up of the same features) or 256
    int nt;             // token rows per tile (TMA box height)
    int k_blocks;
    uint32_t tx_bytes;
    const int32_t* rows;
    void* out;
    int64_t ldo;
    int64_t out_rows_per_group;
    const void* bias;
    int64_t bias_group_stride;
    int vec_ok;
    int32_t* status;
    const __nv_bfloat16* xg;  // gathered mode: token source rows (row stride ldxg)
    int64_t ldxg;
    int64_t kdim;             // K (gathered mode: chunks past K are zero-filled)
    int64_t xrows;            // gathered mode: rows of the source matrix
    const int32_t* gidx;      // gathered mode: (G, max_tokens) source row per token slot
    __nv_bfloat16* save_ab;   // SwiGLU: the pre-activations a (gate) and b (up) in bf16, or NULL
    int64_t ld_save;
};

__device__ __forceinline__ int64_t group_rows(const XParams& p, int g) {
    int64_t r = p.rows ? (int64_t)p.rows[g] : p.max_tokens;
    return r < 0 ? 0 : (r > p.max_tokens ? p.max_tokens : r);
}

// Tile order inside a group: feature tile fastest, so tiles that run together
// share the group's token tile.
__device__ __forceinline__ void decode(int tile, const int* prefix, int G, int f_tiles, int& g, int& ft, int& tt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    g = lo;
    const int local = tile - prefix[g];
    tt = local / f_tiles;
    ft = local - tt * f_tiles;
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(GATHER ? kThreads + kGatherThreads : kThreads, 1)
    tcx_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW2,
               const __grid_constant__ CUtensorMap tmX, const XParams p) {
    constexpr bool kDual = EPI == TC_EPI_SWIGLU;
    constexpr bool kF32 = EPI == TC_EPI_F32;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_prefix[kMaxGroups + 1];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = bars + 2 * kStages;
    uint64_t* tempty = bars + 2 * kStages + 2;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], GATHER ? 1 + kGatherThreads : 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(2 * kAccCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int g = threadIdx.x; g < p.G; g += blockDim.x) {
        const int64_t r = group_rows(p, g);
        s_prefix[g + 1] = (int)((r + p.nt - 1) / p.nt) * p.f_tiles;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        s_prefix[0] = 0;
        for (int g = 0; g < p.G; ++g) s_prefix[g + 1] += s_prefix[g];
    }
    __syncthreads();
    const int total = s_prefix[p.G];
    const uint32_t tmem_base = s_tmem;
    const int x_off = 32 * 1024;  // token tile offset inside a stage

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x) {
                int g, ft, tt;
                decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
                const int32_t w_y = (int32_t)(g * p.w_rows_per_group + (int64_t)ft * p.feat_per_tile);
                const int32_t x_y = (int32_t)(g * p.x_rows_per_group + (int64_t)tt * p.nt);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&full[stage], p.tx_bytes);
                    uint8_t* st = stages + stage * kStageBytes;
                    tma_load_2d(st, &tmW, kb * kBK, w_y, &full[stage]);
                    if (kDual) tma_load_2d(st + 16 * 1024, &tmW2, kb * kBK, w_y, &full[stage]);
                    else tma_load_2d(st + 16 * 1024, &tmW, kb * kBK, w_y + kM, &full[stage]);
                    if (!GATHER) tma_load_2d(st + x_off, &tmX, kb * kBK, x_y, &full[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t it = 0;
            bool ready = false;  // full[stage] was seen complete by an early test
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x, ++it) {
                int g, ft, tt;
                decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
                int64_t n_left = group_rows(p, g) - (int64_t)tt * p.nt;
                if (n_left > p.nt) n_left = p.nt;
                const int n_cur = (int)((n_left + 15) / 16 * 16);
                const uint32_t idesc = make_idesc(kM, n_cur);
                const uint32_t acc = it & 1u;
                const uint32_t acc_phase = (it >> 1) & 1u;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ready && !mbar_wait(&full[stage], phase, p.status)) {
                        s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(stages + stage * kStageBytes);
                    const uint64_t wd = sw128_desc(st);
                    const uint64_t xd = sw128_desc(st + x_off);
                    const int ns = stage + 1 == kStages ? 0 : stage + 1;
                    const uint32_t np = stage + 1 == kStages ? phase ^ 1u : phase;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        tc_mma(d, wd + 2 * kk, xd + 2 * kk, idesc, accum);
                        tc_mma(d + 128, sw128_desc(st + 16 * 1024) + 2 * kk, xd + 2 * kk, idesc, accum);
                        // the tensor core takes new MMAs only as it finishes old ones: look at the
                        // next stage while this one's MMAs are being accepted
                        if (kk == 1) ready = mbar_test(smem_u32(&full[ns]), np);
                    }
                    tc_commit(&empty[stage]);
                    stage = ns;
                    phase = np;
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
            }
        }
        __syncwarp();
    } else if (GATHER && warp >= kThreads / 32) {
        // ------------------------- gathered token rows -------------------------
        // kGatherThreads threads fill the 128 x 64 token tile of each stage with
        // 16-byte cp.async copies from the source rows, in the 128-byte swizzled
        // layout the TMA would produce (chunk j of row r at chunk j ^ (r & 7)).
        // Thread gt copies chunk j = gt & 7 of rows kRowStep*i + (gt >> 3), so
        // eight consecutive threads read one contiguous 128-byte row segment.  A
        // stage is signalled once its copies have landed (kGatherLag stages
        // later), after a proxy fence that makes them visible to the tensor core.
        constexpr int kRowStep = kGatherThreads / 8;
        constexpr int kPasses = kNT / kRowStep;
        const int gt = threadIdx.x - kThreads;
        const int j = gt & 7;
        const int rsub = gt >> 3;
        // row kRowStep*i + rsub has (row & 7) == (rsub & 7) for every i
        const uint32_t dst_off = (uint32_t)(rsub * 128 + ((j ^ (rsub & 7)) << 4));
        int stage = 0;
        uint32_t phase = 0;
        int pending = 0;    // stages issued and not yet signalled
        int sig_stage = 0;  // oldest of them
        bool abort = false;
        for (int tile = blockIdx.x; tile < total && !abort; tile += gridDim.x) {
            int g, ft, tt;
            decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
            const int64_t n0 = (int64_t)tt * p.nt;
            const int64_t rows_g = group_rows(p, g);
            const int32_t* gi = p.gidx + (int64_t)g * p.max_tokens;
            const __nv_bfloat16* src[kPasses];
            uint32_t srcb[kPasses];
#pragma unroll
            for (int i = 0; i < kPasses; ++i) {
                const int64_t n = n0 + kRowStep * i + rsub;
                int32_t t = n < rows_g ? gi[n] : -1;
                if (t >= p.xrows) {  // outside the source matrix: report, read zeros
                    set_status(p.status, MOE_ERR_BAD_INDEX);
                    t = -1;
                }
                src[i] = p.xg + (t >= 0 ? (int64_t)t * p.ldxg : 0) + 8 * j;
                srcb[i] = t >= 0 ? 16u : 0u;
            }
            for (int kb = 0; kb < p.k_blocks; ++kb) {
                int ok = 1;
                if ((threadIdx.x & 31) == 0) ok = mbar_wait(&empty[stage], phase ^ 1u, p.status) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok || s_abort) {
                    s_abort = 1;
                    abort = true;
                    break;
                }
                const uint32_t dst = smem_u32(stages + stage * kStageBytes + x_off) + dst_off;
                const bool in_k = (int64_t)kb * kBK + 8 * j < p.kdim;
#pragma unroll
                for (int i = 0; i < kPasses; ++i)  // a zero-byte copy reads nothing; give it the base address anyway
                    cp_async_16(dst + i * kRowStep * 128, in_k ? src[i] + kb * kBK : p.xg, in_k ? srcb[i] : 0u);
                cp_async_commit();
                ++pending;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (pending > kGatherLag) {
                    cp_async_wait_group<kGatherLag>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full[sig_stage]);
                    sig_stage = sig_stage + 1 == kStages ? 0 : sig_stage + 1;
                    --pending;
                }
            }
        }
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        for (; pending > 0; --pending) {
            mbar_arrive(&full[sig_stage]);
            sig_stage = sig_stage + 1 == kStages ? 0 : sig_stage + 1;
        }
        __syncwarp();
    } else {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int g, ft, tt;
            decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
            const uint32_t acc = it & 1u;
            const uint32_t acc_phase = (it >> 1) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                s_abort = 1;
                break;
            }
            tc_fence_after();
            const int64_t n0 = (int64_t)tt * p.nt;
            int64_t n_valid = group_rows(p, g) - n0;
            if (n_valid > p.nt) n_valid = p.nt;
            const uint32_t t_row = tmem_base + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            const int chunks = (int)((n_valid + 31) / 32);
            // SwiGLU: one output half (gate/up combined); otherwise two halves of 128 features
            for (int half = 0; half < (kDual ? 1 : 2); ++half) {
                const int64_t f0 = (int64_t)ft * p.feat_per_tile + half * kM + 32 * q;  // this warp's first feature
                const int64_t f = f0 + lane;                                            // this thread's feature
                float bias_f = 0.f;
                if (p.bias && f < p.features) {
                    if (kF32) bias_f = reinterpret_cast<const float*>(p.bias)[f];
                    else
                        bias_f = __bfloat162float(
                            reinterpret_cast<const __nv_bfloat16*>(p.bias)[g * p.bias_group_stride + f]);
                }
                const uint32_t t_acc = t_row + half * 128;
                for (int c = 0; c < chunks; ++c) {
                    uint32_t r[32];
                    tmem_ld32(t_acc + c * 32, r);
                    tmem_ld_wait(r);
                    float o[32];
                    if (kDual) {
                        uint32_t u[32];
                        tmem_ld32(t_row + 128 + c * 32, u);
                        tmem_ld_wait(u);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = silu_f(__uint_as_float(r[i])) * __uint_as_float(u[i]);
                        if (p.save_ab && f < p.features) {  // [a | b] rows for the backward
                            const int64_t row0 = (int64_t)g * p.out_rows_per_group + n0 + c * 32;
                            const int i_end = (int)((n_valid - c * 32) < 32 ? (n_valid - c * 32) : 32);
                            __nv_bfloat16* sa = p.save_ab + row0 * p.ld_save + f;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < i_end) {
                                    sa[(int64_t)i * p.ld_save] = __float2bfloat16_rn(__uint_as_float(r[i]));
                                    sa[(int64_t)i * p.ld_save + p.features] = __float2bfloat16_rn(__uint_as_float(u[i]));
                                }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            float v = __uint_as_float(r[i]) + bias_f;
                            if (EPI == TC_EPI_GELU_BIAS) v = gelu_f(v);
                            o[i] = v;
                        }
                    }
                    // Store: for each of the 32 tokens the warp writes 32 consecutive
                    // features of that token's row (one contiguous run per instruction).
                    if (f < p.features) {
                        const int64_t row0 = (int64_t)g * p.out_rows_per_group + n0 + c * 32;
                        const int i_end = (int)((n_valid - c * 32) < 32 ? (n_valid - c * 32) : 32);
                        if (kF32) {
                            float* dst = reinterpret_cast<float*>(p.out) + row0 * p.ldo + f;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < i_end) dst[(int64_t)i * p.ldo] = o[i];
                        } else {
                            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + row0 * p.ldo + f;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < i_end) dst[(int64_t)i * p.ldo] = __float2bfloat16_rn(o[i]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (s_abort) break;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kAccCols)
                     : "memory");
    }
}

template <int EPI, bool GATHER = false>
int launch(const CUtensorMap& w, const CUtensorMap& w2, const CUtensorMap& x, const XParams& kp, int grid,
           cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 64 || !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(tcx_kernel<EPI, GATHER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kSmemBytes));
        if (dev < 64) attr_set[dev] = true;
    }
    tcx_kernel<EPI, GATHER><<<grid, GATHER ? kThreads + kGatherThreads : kThreads, kSmemBytes, stream>>>(w, w2, x,
                                                                                                         kp);
    return launch_status();
}

}  // namespace

int tcx_gemm_run(const TcxProblem& p, cudaStream_t stream) {
    const bool dual = p.epilogue == TC_EPI_SWIGLU;
    MOE_REQUIRE(p.w && p.x && p.out && (!dual || p.w2), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G >= 1 && p.features >= 1 && p.max_tokens >= 0 && p.K >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G <= kMaxGroups, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(aligned16(p.w) && aligned16(p.x) && (!dual || aligned16(p.w2)) && (p.ldw * 2) % 16 == 0 &&
                    (p.ldx * 2) % 16 == 0,
                MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(p.ldw >= p.K && p.ldx >= p.K, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.w_rows_total < (int64_t(1) << 31) && p.x_rows_total < (int64_t(1) << 31), MOE_ERR_UNSUPPORTED);
    const bool gather = p.gather_index != nullptr;
    if (gather) MOE_REQUIRE(dual && p.K % 8 == 0, MOE_ERR_UNSUPPORTED);
    if (p.max_tokens == 0) return MOE_OK;

    XParams kp{};
    kp.G = p.G;
    kp.w_rows_per_group = p.w_rows_per_group;
    kp.x_rows_per_group = p.x_rows_per_group;
    kp.features = p.features;
    kp.max_tokens = p.max_tokens;
    kp.feat_per_tile = dual ? kM : 2 * kM;
    kp.f_tiles = (int)((p.features + kp.feat_per_tile - 1) / kp.feat_per_tile);
    kp.nt = kNT;
    kp.k_blocks = (int)((p.K + kBK - 1) / kBK);
    kp.tx_bytes = (uint32_t)(2 * kM * kBK * 2 + (gather ? 0 : kp.nt * kBK * 2));
    kp.rows = p.rows;
    kp.out = p.out;
    kp.ldo = p.ldo;
    kp.save_ab = static_cast<__nv_bfloat16*>(p.save_ab);
    kp.ld_save = p.ld_save;
    kp.out_rows_per_group = p.out_rows_per_group;
    kp.bias = p.bias;
    kp.bias_group_stride = p.bias_group_stride;
    const size_t esz = p.epilogue == TC_EPI_F32 ? 4 : 2;
    kp.vec_ok = aligned16(p.out) && (p.ldo * (int64_t)esz) % 16 == 0;
    kp.status = p.status;
    kp.xg = static_cast<const __nv_bfloat16*>(p.x);
    kp.ldxg = p.ldx;
    kp.kdim = p.K;
    kp.gidx = p.gather_index;
    kp.xrows = p.x_rows_total;

    CUtensorMap mw, mw2, mx;
    MOE_REQUIRE(make_map(&mw, p.w, p.K, p.w_rows_total, p.ldw, kM), MOE_ERR_CUDA);
    if (dual) MOE_REQUIRE(make_map(&mw2, p.w2, p.K, p.w_rows_total, p.ldw, kM), MOE_ERR_CUDA);
    else mw2 = mw;
    if (gather) mx = mw;  // token rows are copied by the kernel's gather warps
    else MOE_REQUIRE(make_map(&mx, p.x, p.K, p.x_rows_total, p.ldx, kp.nt), MOE_ERR_CUDA);

    const int64_t max_tiles = (int64_t)p.G * kp.f_tiles * ((p.max_tokens + kp.nt - 1) / kp.nt);
    MOE_REQUIRE(max_tiles < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    int grid = device_sm_count();
    if (max_tiles < grid) grid = (int)max_tiles;
    if (grid < 1) grid = 1;

    // The library uses this kernel for the SwiGLU gate/up projection only.
    if (p.epilogue != TC_EPI_SWIGLU) return MOE_ERR_UNSUPPORTED;
    return gather ? launch<TC_EPI_SWIGLU, true>(mw, mw2, mx, kp, grid, stream)
                  : launch<TC_EPI_SWIGLU>(mw, mw2, mx, kp, grid, stream);
}

}  // namespace moe
