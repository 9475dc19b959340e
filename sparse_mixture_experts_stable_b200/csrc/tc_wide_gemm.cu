// Grouped SwiGLU gate/up GEMM over the routed experts, 256 features x up to
// 256 tokens per tile, on pairs of SMs:
//
//   h[g, n, f] = silu( sum_k Wg[g, f, k] X[g, n, k] ) * ( sum_k Wu[g, f, k] X[g, n, k] )      n < rows[g]
//
// Why this shape.  One SM's tensor core consumes 8192 bf16 FLOP per clock, and
// the operands reach its shared memory through the TMA.  Two CTAs on two SMs
// (a cluster) share each tcgen05 MMA of M = 256 features x N tokens: each CTA
// stages the gate and up rows of its own 128 features and half of the tile's
// token rows, and its tensor memory receives its 128 features x all N tokens.
// Per 64-deep K block that is 48 KB per SM (16 KB gate, 16 KB up, 16 KB of
// tokens) for 2 x 128 x 256 x 64 MACs, against 64 KB for the same work on one
// SM, and four stages fit in shared memory where three did.  The two fp32
// accumulators (gate and up, 128 x 256 each) fill all 512 TMEM columns, so
// TMEM is single-buffered: the epilogue first drains the accumulators into
// registers (silu(g)*u packed to bf16, a cheap exponential), releases TMEM so
// the next tile's MMAs start, and only then stores.  A ragged expert sets N per
// tile (its tokens split in two halves rounded up to 16) and loads only the
// 32-row boxes holding them.
//
// Warp roles (576 threads per CTA, one persistent CTA per SM):
//   warp 0      TMA producer: 4 stages of [gate 128 x 64 | up 128 x 64 | N/2 tokens x 64].
//               The even CTA's producer draws the tiles (one global counter, so
//               pairs that drew short tiles take more) and hands each index to
//               both CTAs through a small queue; it arms each stage's barrier
//               with the bytes of both CTAs, whose loads all land on it.
//   warp 1      TMEM owner (512 columns, both CTAs) and MMA issuer (one lane of
//               the even CTA)
//   warps 2-17  epilogue: warp w drains TMEM lanes 32*(w%4).. (32 features of
//               each accumulator) for the 64 tokens [64*r, 64*r + 64), r = (w - 2) / 4
// Every mbarrier wait is bounded (kWaitLimitNs).  After a timeout the producer
// and the MMA issuer stop; the epilogue keeps walking its tiles (each wait
// bounded) without writing, so the kernel always reaches its closing cluster
// barrier.
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

constexpr int kM = 128;        // features per CTA (half of the pair's UMMA M = 256)
constexpr int kBK = 64;        // K per stage
constexpr int kNT = 256;       // max tokens per tile (UMMA N)
constexpr int kBox = 32;       // token rows per TMA box
constexpr int kStages = 4;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kMaxGroups = 1024;
constexpr int kQueue = 4;      // tile indices in flight between the producer and the consumers
constexpr int kWBytes = kM * kBK * 2;                 // 16 KB per weight tile
constexpr int kXBytes = (kNT / 2) * kBK * 2;          // 16 KB: this CTA's half of the tokens
constexpr int kStageBytes = 2 * kWBytes + kXBytes;    // 48 KB
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;
// consumers of a queue slot, all counted on the even CTA: its MMA issuer and
// epilogue warps, the odd CTA's producer and epilogue warps
constexpr int kQueueConsumers = 1 + kEpiWarps + 1 + kEpiWarps;

struct WParams {
    int G;
    int64_t w_rows_per_group;
    int64_t x_rows_per_group;
    int64_t features;
    int64_t max_tokens;
    int f_tiles;  // tiles of 256 features
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

// the tokens of one CTA: a tile's n_valid tokens in two halves of `half` rows
// (a multiple of 16, so N = 2 * half is a valid MMA width)
__device__ __forceinline__ int token_half(int64_t n_valid) { return (int)(((n_valid + 1) / 2 + 15) / 16 * 16); }

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

// silu(a) * b = a * sigmoid(a) * b with sigmoid(a) = 1/2 + tanh(a/2)/2 through the
// hardware tanh approximation (tanh.approx.f32, relative error about 2^-11): one
// special-function operation per element where exp and a reciprocal took two, and
// the drain of the accumulators, which holds up the next tile's MMAs, is bound by
// that unit.  The product is rounded to bf16 (spacing 2^-8 relative).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float swiglu_fast(float a, float b) {
    return a * fmaf(0.5f, tanh_approx(0.5f * a), 0.5f) * b;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, int v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tcw_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
               const __grid_constant__ CUtensorMap tmX, const WParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_prefix[kMaxGroups + 1];
    __shared__ int s_tile[kQueue];  // tiles handed out to this pair, in order
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full = bars;                // even CTA: a stage's loads of both CTAs have landed
    uint64_t* empty = bars + kStages;     // both CTAs: the stage's MMAs are done
    uint64_t* tfull = bars + 2 * kStages; // both CTAs: the accumulators hold a finished tile
    uint64_t* tempty = tfull + 1;         // even CTA: both epilogues drained the accumulators
    uint64_t* qfull = tempty + 1;         // both CTAs: s_tile[q] holds the next tile
    uint64_t* qempty = qfull + kQueue;    // even CTA: every consumer has read s_tile[q]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 2 * kEpiWarps);
        for (int q = 0; q < kQueue; ++q) {
            mbar_init(&qfull[q], 1);
            mbar_init(&qempty[q], kQueueConsumers);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmWg)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmWu)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    for (int g = threadIdx.x; g < p.G; g += blockDim.x) {
        const int64_t r = group_rows(p, g);
        s_prefix[g + 1] = r > 0 ? (int)((r + token_span(r) - 1) / token_span(r)) * p.f_tiles : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s_prefix[0] = 0;
        for (int g = 0; g < p.G; ++g) s_prefix[g + 1] += s_prefix[g];
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
    tc_fence_after();
    const int total = s_prefix[p.G];
    const uint32_t tmem_base = s_tmem;
    // the even CTA's barriers as shared::cluster addresses
    const uint32_t full_l = mapa_shared(smem_u32(full), 0);
    const uint32_t tempty_l = mapa_shared(smem_u32(tempty), 0);
    const uint32_t qempty_l = mapa_shared(smem_u32(qempty), 0);

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0;; ++i) {
                const int q = i % kQueue;
                const uint32_t qph = (uint32_t)(i / kQueue) & 1u;
                int tile;
                if (leader) {
                    if (!mbar_wait_cluster(&qempty[q], qph ^ 1u, p.status)) {
                        s_abort = 1;
                        tile = -1;
                    } else {
                        tile = s_abort ? -1 : (int)atomicAdd(p.tile_counter, 1u);
                        if (tile >= total) tile = -1;
                    }
                    s_tile[q] = tile;
                    st_cluster_u32(mapa_shared(smem_u32(&s_tile[q]), 1), tile);
                    mbar_arrive(&qfull[q]);
                    mbar_arrive_cluster(mapa_shared(smem_u32(&qfull[q]), 1));  // release: orders the store
                } else {
                    tile = -1;
                    if (mbar_wait_cluster(&qfull[q], qph, p.status)) tile = s_tile[q];
                    else s_abort = 1;
                    mbar_arrive_cluster(qempty_l + 8u * (uint32_t)q);
                }
                if (tile < 0) break;
                int g, ft, tt;
                decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
                int64_t n0, n_valid;
                token_range(p, g, tt, n0, n_valid);
                const int half = token_half(n_valid);
                const int nbox = (half + kBox - 1) / kBox;
                const int32_t w_y = (int32_t)(g * p.w_rows_per_group + (int64_t)ft * 2 * kM + (int64_t)rank * kM);
                const int32_t x_y = (int32_t)(g * p.x_rows_per_group + n0 + (int64_t)rank * half);
                const uint32_t tx_pair = 2u * (uint32_t)(2 * kWBytes + nbox * kBox * kBK * 2);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    if (leader) mbar_expect_tx(&full[stage], tx_pair);
                    const uint32_t fb = full_l + 8u * (uint32_t)stage;
                    uint8_t* st = smem + stage * kStageBytes;
                    tma_load_2d_pair(st, &tmWg, kb * kBK, w_y, fb);
                    tma_load_2d_pair(st + kWBytes, &tmWu, kb * kBK, w_y, fb);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d_pair(st + 2 * kWBytes + b * (kBox * kBK * 2), &tmX, kb * kBK, x_y + b * kBox, fb);
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
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            bool ready = false;  // full[stage] was seen complete by an early test
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
                int64_t n0, n_valid;
                token_range(p, g, tt, n0, n_valid);
                const uint32_t idesc = make_idesc(2 * kM, 2 * token_half(n_valid));
                if (!mbar_wait_cluster(tempty, (it & 1u) ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ready && !mbar_wait(&full[stage], phase, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * kStageBytes);
                    const uint64_t gd = sw128_desc(st), ud = sw128_desc(st + kWBytes);
                    const uint64_t xd = sw128_desc(st + 2 * kWBytes);
                    const int ns = stage + 1 == kStages ? 0 : stage + 1;
                    const uint32_t np = stage + 1 == kStages ? phase ^ 1u : phase;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        tc_mma_pair(tmem_base, gd + 2 * kk, xd + 2 * kk, idesc, accum);
                        tc_mma_pair(tmem_base + 256, ud + 2 * kk, xd + 2 * kk, idesc, accum);
                        // the tensor core takes new MMAs only as it finishes old ones: look at the
                        // next stage while this one's MMAs are being accepted
                        if (kk == 1) ready = mbar_test(smem_u32(&full[ns]), np);
                    }
                    tc_commit_pair(&empty[stage]);
                    stage = ns;
                    phase = np;
                }
                if (!ok) {
                    s_abort = 1;
                    break;
                }
                tc_commit_pair(tfull);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;          // TMEM lane quarter: features 32q .. 32q+31 of this CTA's 128
        const int r = (warp - 2) >> 2;   // token quarter: tokens 64r .. 64r+63 of the tile
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        for (uint32_t it = 0;; ++it) {
            const int q_slot = (int)(it % kQueue);
            int tile = -1;
            if (lane == 0) {
                if (mbar_wait_cluster(&qfull[q_slot], (it / kQueue) & 1u, p.status)) tile = s_tile[q_slot];
                else s_abort = 1;
                mbar_arrive_cluster(qempty_l + 8u * (uint32_t)q_slot);
            }
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (tile < 0) break;
            int g, ft, tt;
            decode(tile, s_prefix, p.G, p.f_tiles, g, ft, tt);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(tfull, it & 1u, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) s_abort = 1;
            tc_fence_after();
            int64_t n0, n_valid;
            token_range(p, g, tt, n0, n_valid);
            // this thread's feature
            const int64_t f = (int64_t)ft * 2 * kM + (int64_t)rank * kM + q * 32 + lane;
            const bool live = !s_abort;
            const int64_t row0 = (int64_t)g * p.out_rows_per_group + n0 + 64 * r;
            uint32_t hp[4][8];  // this warp's 64 tokens as bf16 pairs

            // drain this warp's 64 tokens, 16 at a time: gate and up -> silu(g)*u
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int tok0 = 64 * r + 16 * ch;
                if (tok0 < n_valid) {
                    uint32_t ga[16], up[16];
                    tmem_ld16(tmem_base + lane_off + (uint32_t)tok0, ga);
                    tmem_ld16(tmem_base + 256 + lane_off + (uint32_t)tok0, up);
                    tmem_ld_wait(ga, up);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        hp[ch][i] = pack_bf16x2(swiglu_fast(__uint_as_float(ga[2 * i]), __uint_as_float(up[2 * i])),
                                                swiglu_fast(__uint_as_float(ga[2 * i + 1]), __uint_as_float(up[2 * i + 1])));
                    if (p.save_ab && live && f < p.features) {  // the pre-activations [a | b] for the backward
                        const int i_end = (int)(n_valid - tok0 < 16 ? n_valid - tok0 : 16);
                        __nv_bfloat16* sa = p.save_ab + (row0 + 16 * ch) * p.ld_save + f;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (i < i_end) {
                                sa[(int64_t)i * p.ld_save] = __float2bfloat16_rn(__uint_as_float(ga[i]));
                                sa[(int64_t)i * p.ld_save + p.features] = __float2bfloat16_rn(__uint_as_float(up[i]));
                            }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_l);  // TMEM drained: the next tile's MMAs may start
            // store: for each token the warp writes 32 consecutive features (one 64-byte run)
            if (live && f < p.features) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int tok0 = 64 * r + 16 * ch;
                    const int i_end = (int)(n_valid - tok0 < 0 ? 0 : (n_valid - tok0 < 16 ? n_valid - tok0 : 16));
                    __nv_bfloat16* dst = p.out + (row0 + 16 * ch) * p.ldo + f;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (i < i_end) {
                            const uint32_t w = hp[ch][i >> 1];
                            dst[(int64_t)i * p.ldo] =
                                __ushort_as_bfloat16((i & 1) ? (uint16_t)(w >> 16) : (uint16_t)(w & 0xFFFFu));
                        }
                }
            }
        }
    }

    tc_fence_before();
    cluster_sync();  // neither CTA leaves while the other may still signal its barriers or read its stages
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
    }
}

int launch_tcw(const CUtensorMap& mg, const CUtensorMap& mu, const CUtensorMap& mx, const WParams& kp, int grid,
               cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 64 || !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(tcw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes));
        if (dev < 64) attr_set[dev] = true;
    }
    tcw_kernel<<<grid, kThreads, kSmemBytes, stream>>>(mg, mu, mx, kp);
    return launch_status();
}

}  // namespace

int tcw_gemm_run(const TcxProblem& p, cudaStream_t stream) {
    MOE_REQUIRE(p.epilogue == TC_EPI_SWIGLU && p.gather_index == nullptr && p.bias == nullptr, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(p.w && p.w2 && p.x && p.out && p.tile_counter, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G >= 1 && p.features >= 1 && p.max_tokens >= 0 && p.K >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G <= kMaxGroups, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(aligned16(p.w) && aligned16(p.w2) && aligned16(p.x) && (p.ldw * 2) % 16 == 0 && (p.ldx * 2) % 16 == 0,
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
    kp.f_tiles = (int)((p.features + 2 * kM - 1) / (2 * kM));
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
    MOE_REQUIRE(make_map(&mu, p.w2, p.K, p.w_rows_total, p.ldw, kM), MOE_ERR_CUDA);
    MOE_REQUIRE(make_map(&mx, p.x, p.K, p.x_rows_total, p.ldx, kBox), MOE_ERR_CUDA);

    const int64_t max_tiles = (int64_t)p.G * kp.f_tiles * ((p.max_tokens + kNT - 1) / kNT);  // upper bound
    MOE_REQUIRE(max_tiles < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    int64_t pairs = device_sm_count() / 2;
    if (max_tiles < pairs) pairs = max_tiles;
    if (pairs < 1) pairs = 1;
    return launch_tcw(mg, mu, mx, kp, (int)(2 * pairs), stream);
}

}  // namespace moe
