// Grouped expert GEMMs with 256 weight rows x up to 256 tokens per tile.
//
//   SwiGLU gate/up: h[g, n, f] = silu( sum_k Wg[g, f, k] X[g, n, k] ) * ( sum_k Wu[g, f, k] X[g, n, k] )
//   plain (down):   y[g, n, f] = sum_k W[g, f, k] X[g, n, k]                            n < rows[g]
//
// Why this shape.  On this part the TMA brings at most about 72 bytes per clock
// into one SM's shared memory from L2 (measured), while one SM's tensor cores
// consume 8192 bf16 FLOP per clock.  A tile of 256 weight rows x 128 tokens
// (two M=128 MMAs sharing the token operand) needs 48 KB per 64-deep K block,
// 96 bytes per clock at full MMA rate, so it cannot get past ~3/4 of the MMA
// rate; 256 weight rows (gate and up of 128 features) x 256 tokens need 64 KB
// per K block for twice the work, 62.5 bytes per clock, under the TMA ceiling.
// The price: the two fp32 accumulators (gate and up, 128 x 256 each) fill all
// 512 TMEM columns, so TMEM is single-buffered.  The epilogue therefore first
// drains the accumulators into registers (gate and up -> silu(g)*u packed to
// bf16, a cheap exponential), releases TMEM so the next tile's MMAs start, and
// only then stores; the bubble is the drain, a few percent of a K = 2048 tile.
//
// The down projection (K = 512) uses the same tile with two consecutive blocks
// of 128 output features as the two MMAs' A operands; its drain is a larger
// share of its short K loop.  A ragged expert sets N per tile (its remaining
// tokens rounded up to 16, at most 256) and loads only the 32-row boxes holding
// its tokens.
//
// Warp roles (576 threads, one persistent CTA per SM):
//   warp 0      TMA producer: 3 stages of [A0 128 x 64 | A1 128 x 64 | 256 tokens x 64]
//               (A0, A1 = gate and up rows of 128 features, or rows f..f+127 and
//               f+128..f+255 of one weight)
//   warp 1      TMEM owner (512 columns) and MMA issuer (one lane)
//   warps 2-17  epilogue: warp w drains TMEM lanes 32*(w%4).. (32 weight rows of
//               each MMA) for the 64 tokens [64*r, 64*r + 64), r = (w - 2) / 4
// Every mbarrier wait is bounded (kWaitLimitNs).  After a timeout the producer
// and the MMA issuer stop; the epilogue keeps walking its tiles (each wait
// bounded) without writing, so the kernel always ends.
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

constexpr int kM = 128;        // features per tile (UMMA M of each of the two MMAs)
constexpr int kBK = 64;        // K per stage
constexpr int kNT = 256;       // max tokens per tile (UMMA N)
constexpr int kBox = 32;       // token rows per TMA box
constexpr int kStages = 3;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kMaxGroups = 1024;
constexpr int kQueue = 4;      // tile indices in flight between the producer and the consumers
constexpr int kWBytes = kM * kBK * 2;                 // 16 KB per weight tile
constexpr int kXBytes = kNT * kBK * 2;                // 32 KB token tile
constexpr int kStageBytes = 2 * kWBytes + kXBytes;    // 64 KB
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

struct WParams {
    int G;
    int64_t w_rows_per_group;
    int64_t x_rows_per_group;
    int64_t features;
    int64_t max_tokens;
    int f_tiles;
    int feat_per_tile;  // 128 (SwiGLU: gate and up of the same features) or 256
    int k_blocks;
    const int32_t* rows;
    __nv_bfloat16* out;
    int64_t ldo;
    int64_t out_rows_per_group;
    __nv_bfloat16* save_ab;
    int64_t ld_save;
    uint32_t* tile_counter;  // zero at launch: the next tile to hand out
    int32_t* status;
};

__device__ __forceinline__ int64_t group_rows(const WParams& p, int g) {
    int64_t r = p.rows ? (int64_t)p.rows[g] : p.max_tokens;
    return r < 0 ? 0 : (r > p.max_tokens ? p.max_tokens : r);
}

// A group's tokens split into ceil(rows / 256) tiles of equal size (a multiple
// of 32, the TMA box): tile tt covers [tt * span, min((tt + 1) * span, rows)).
__device__ __forceinline__ int64_t token_span(int64_t rows) {
    const int64_t n_tt = (rows + kNT - 1) / kNT;
    if (n_tt <= 0) return kNT;
    const int64_t span = (rows + n_tt - 1) / n_tt;
    return (span + kBox - 1) / kBox * kBox;
}

__device__ __forceinline__ void token_range(const WParams& p, int g, int tt, int64_t& n0, int64_t& n_valid) {
    const int64_t rows = group_rows(p, g);
    const int64_t span = token_span(rows);
    n0 = (int64_t)tt * span;
    n_valid = rows - n0 < span ? rows - n0 : span;
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

// silu(a) * b with a fast exponential: the product is rounded to bf16, whose
// spacing (2^-8 relative) is far above the exponential's error.
__device__ __forceinline__ float swiglu_fast(float a, float b) { return __fdividef(a, 1.0f + __expf(-a)) * b; }

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tcw_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
               const __grid_constant__ CUtensorMap tmX, const WParams p) {
    constexpr bool kSwiglu = EPI == TC_EPI_SWIGLU;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_prefix[kMaxGroups + 1];
    __shared__ int s_tile[kQueue];  // tiles handed out to this CTA, in order
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = bars + 2 * kStages;
    uint64_t* tempty = tfull + 1;
    uint64_t* qfull = tempty + 1;
    uint64_t* qempty = qfull + kQueue;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, kEpiWarps * 32);
        for (int q = 0; q < kQueue; ++q) {
            mbar_init(&qfull[q], 1);
            mbar_init(&qempty[q], 1 + kEpiWarps);  // the MMA issuer and one lane per epilogue warp
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmWg)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmWu)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int g = threadIdx.x; g < p.G; g += blockDim.x) {
        const int64_t r = group_rows(p, g);
        s_prefix[g + 1] = r > 0 ? (int)((r + token_span(r) - 1) / token_span(r)) * p.f_tiles : 0;
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

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        // Tiles are handed out dynamically (one global counter), so CTAs that drew
        // short tiles take more of them; each index goes through a small queue to
        // the MMA issuer and the epilogue warps.  -1 ends the walk.
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0;; ++i) {
                const int q = i % kQueue;
                const uint32_t qph = (uint32_t)(i / kQueue) & 1u;
                if (!mbar_wait(&qempty[q], qph ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                int tile = s_abort ? -1 : (int)atomicAdd(p.tile_counter, 1u);
                if (tile >= total) tile = -1;
                s_tile[q] = tile;
                mbar_arrive(&qfull[q]);
                if (tile < 0) break;
                int g, ft, tt;
                decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
                int64_t n0, n_valid;
                token_range(p, g, tt, n0, n_valid);
                const int nbox = (int)((n_valid + kBox - 1) / kBox);
                const int32_t w_y = (int32_t)(g * p.w_rows_per_group + (int64_t)ft * p.feat_per_tile);
                const int32_t x_y = (int32_t)(g * p.x_rows_per_group + n0);
                const uint32_t tx = (uint32_t)(2 * kWBytes + nbox * kBox * kBK * 2);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&full[stage], tx);
                    uint8_t* st = smem + stage * kStageBytes;
                    tma_load_2d(st, &tmWg, kb * kBK, w_y, &full[stage]);
                    if (kSwiglu) tma_load_2d(st + kWBytes, &tmWu, kb * kBK, w_y, &full[stage]);
                    else tma_load_2d(st + kWBytes, &tmWg, kb * kBK, w_y + kM, &full[stage]);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(st + 2 * kWBytes + b * (kBox * kBK * 2), &tmX, kb * kBK, x_y + b * kBox,
                                    &full[stage]);
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
            for (uint32_t it = 0;; ++it) {
                const int q = (int)(it % kQueue);
                if (!mbar_wait(&qfull[q], (it / kQueue) & 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                const int tile = s_tile[q];
                mbar_arrive(&qempty[q]);
                if (tile < 0) break;
                int g, ft, tt;
                decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
                int64_t n0, n_left;
                token_range(p, g, tt, n0, n_left);
                const int n_cur = (int)((n_left + 15) / 16 * 16);
                const uint32_t idesc = make_idesc(kM, n_cur);
                if (!mbar_wait(tempty, (it & 1u) ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * kStageBytes);
                    const uint64_t gd = sw128_desc(st), ud = sw128_desc(st + kWBytes);
                    const uint64_t xd = sw128_desc(st + 2 * kWBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        tc_mma(tmem_base, gd + 2 * kk, xd + 2 * kk, idesc, accum);
                        tc_mma(tmem_base + 256, ud + 2 * kk, xd + 2 * kk, idesc, accum);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) {
                    s_abort = 1;
                    break;
                }
                tc_commit(tfull);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;          // TMEM lane quarter: features 32q .. 32q+31 of the tile
        const int r = (warp - 2) >> 2;   // token quarter: tokens 64r .. 64r+63 of the tile
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        for (uint32_t it = 0;; ++it) {
            const int q_slot = (int)(it % kQueue);
            int tile = -1;
            if (lane == 0) {
                if (mbar_wait(&qfull[q_slot], (it / kQueue) & 1u, p.status)) tile = s_tile[q_slot];
                else s_abort = 1;
                mbar_arrive(&qempty[q_slot]);
            }
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (tile < 0) break;
            int g, ft, tt;
            decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(tfull, it & 1u, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                s_abort = 1;
                break;
            }
            tc_fence_after();
            int64_t n0, n_valid;
            token_range(p, g, tt, n0, n_valid);
            const int64_t f = (int64_t)ft * p.feat_per_tile + q * 32 + lane;  // this thread's first feature
            const bool live = !s_abort;
            const int64_t row0 = (int64_t)g * p.out_rows_per_group + n0 + 64 * r;
            constexpr int NA = kSwiglu ? 1 : 2;  // output blocks of 128 features per tile
            uint32_t hp[4][8];                   // one block's 64 tokens as bf16 pairs

#pragma unroll
            for (int a = 0; a < NA; ++a) {
                // drain this warp's 64 tokens, 16 at a time (SwiGLU: gate and up -> silu(g)*u)
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int tok0 = 64 * r + 16 * ch;
                    if (tok0 < n_valid) {
                        if (kSwiglu) {
                            uint32_t ga[16], up[16];
                            tmem_ld16(tmem_base + lane_off + (uint32_t)tok0, ga);
                            tmem_ld16(tmem_base + 256 + lane_off + (uint32_t)tok0, up);
                            tmem_ld_wait(ga, up);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                hp[ch][i] = pack_bf16x2(
                                    swiglu_fast(__uint_as_float(ga[2 * i]), __uint_as_float(up[2 * i])),
                                    swiglu_fast(__uint_as_float(ga[2 * i + 1]), __uint_as_float(up[2 * i + 1])));
                            if (p.save_ab && live && f < p.features) {  // the pre-activations [a | b] for the backward
                                const int i_end = (int)(n_valid - tok0 < 16 ? n_valid - tok0 : 16);
                                __nv_bfloat16* sa = p.save_ab + (row0 + 16 * ch) * p.ld_save + f;
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    if (i < i_end) {
                                        sa[(int64_t)i * p.ld_save] = __float2bfloat16_rn(__uint_as_float(ga[i]));
                                        sa[(int64_t)i * p.ld_save + p.features] =
                                            __float2bfloat16_rn(__uint_as_float(up[i]));
                                    }
                            }
                        } else {
                            uint32_t v[16], unused[16];
                            tmem_ld16(tmem_base + 256 * a + lane_off + (uint32_t)tok0, v);
                            tmem_ld_wait(v, unused);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                hp[ch][i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        }
                    }
                }
                if (a == NA - 1) {
                    tc_fence_before();
                    mbar_arrive(tempty);  // TMEM drained: the next tile's MMAs may start
                }
                // store: for each token the warp writes 32 consecutive features (one 64-byte run)
                const int64_t fa = f + a * kM;
                if (live && fa < p.features) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int tok0 = 64 * r + 16 * ch;
                        const int i_end =
                            (int)(n_valid - tok0 < 0 ? 0 : (n_valid - tok0 < 16 ? n_valid - tok0 : 16));
                        __nv_bfloat16* dst = p.out + (row0 + 16 * ch) * p.ldo + fa;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (i < i_end) {
                                const uint32_t w = hp[ch][i >> 1];
                                dst[(int64_t)i * p.ldo] = __ushort_as_bfloat16((i & 1) ? (uint16_t)(w >> 16)
                                                                                       : (uint16_t)(w & 0xFFFFu));
                            }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
    }
}

}  // namespace

namespace {

template <int EPI>
int launch_tcw(const CUtensorMap& mg, const CUtensorMap& mu, const CUtensorMap& mx, const WParams& kp, int grid,
               cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 64 || !attr_set[dev]) {
        MOE_CUDA_TRY(
            cudaFuncSetAttribute(tcw_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes));
        if (dev < 64) attr_set[dev] = true;
    }
    tcw_kernel<EPI><<<grid, kThreads, kSmemBytes, stream>>>(mg, mu, mx, kp);
    return launch_status();
}

}  // namespace

int tcw_gemm_run(const TcxProblem& p, cudaStream_t stream) {
    const bool swiglu = p.epilogue == TC_EPI_SWIGLU;
    MOE_REQUIRE((swiglu || p.epilogue == TC_EPI_BF16) && p.gather_index == nullptr && p.bias == nullptr,
                MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(p.w && p.x && p.out && (!swiglu || p.w2) && p.tile_counter, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(swiglu || p.save_ab == nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G >= 1 && p.features >= 1 && p.max_tokens >= 0 && p.K >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G <= kMaxGroups, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(aligned16(p.w) && (!swiglu || aligned16(p.w2)) && aligned16(p.x) && (p.ldw * 2) % 16 == 0 &&
                    (p.ldx * 2) % 16 == 0,
                MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(p.ldw >= p.K && p.ldx >= p.K, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.w_rows_total < (int64_t(1) << 31) && p.x_rows_total < (int64_t(1) << 31), MOE_ERR_UNSUPPORTED);
    if (p.max_tokens == 0) return MOE_OK;

    WParams kp{};
    kp.G = p.G;
    kp.w_rows_per_group = p.w_rows_per_group;
    kp.x_rows_per_group = p.x_rows_per_group;
    kp.features = p.features;
    kp.max_tokens = p.max_tokens;
    kp.feat_per_tile = swiglu ? kM : 2 * kM;
    kp.f_tiles = (int)((p.features + kp.feat_per_tile - 1) / kp.feat_per_tile);
    kp.k_blocks = (int)((p.K + kBK - 1) / kBK);
    kp.rows = p.rows;
    kp.out = static_cast<__nv_bfloat16*>(p.out);
    kp.ldo = p.ldo;
    kp.out_rows_per_group = p.out_rows_per_group;
    kp.save_ab = static_cast<__nv_bfloat16*>(p.save_ab);
    kp.ld_save = p.ld_save;
    kp.tile_counter = p.tile_counter;
    kp.status = p.status;
    MOE_CUDA_TRY(cudaMemsetAsync(p.tile_counter, 0, sizeof(uint32_t), stream));

    CUtensorMap mg, mu, mx;
    MOE_REQUIRE(make_map(&mg, p.w, p.K, p.w_rows_total, p.ldw, kM), MOE_ERR_CUDA);
    if (swiglu) MOE_REQUIRE(make_map(&mu, p.w2, p.K, p.w_rows_total, p.ldw, kM), MOE_ERR_CUDA);
    else mu = mg;
    MOE_REQUIRE(make_map(&mx, p.x, p.K, p.x_rows_total, p.ldx, kBox), MOE_ERR_CUDA);

    const int64_t max_tiles = (int64_t)p.G * kp.f_tiles * ((p.max_tokens + kNT - 1) / kNT);  // upper bound
    MOE_REQUIRE(max_tiles < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    int grid = device_sm_count();
    if (max_tiles < grid) grid = (int)max_tiles;
    if (grid < 1) grid = 1;
    return swiglu ? launch_tcw<TC_EPI_SWIGLU>(mg, mu, mx, kp, grid, stream)
                  : launch_tcw<TC_EPI_BF16>(mg, mu, mx, kp, grid, stream);
}

}  // namespace moe
