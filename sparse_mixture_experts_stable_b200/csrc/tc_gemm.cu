// Grouped bf16 GEMM on sm_100a: TMA (128B swizzle) -> shared memory ->
// tcgen05.mma (kind::f16, fp32 accumulate in TMEM) -> tcgen05.ld -> epilogue.
//
// Warp roles in a 192-thread persistent CTA (one per SM):
//   warp 0      : TMA producer (one lane), 4-stage smem ring
//   warp 1      : TMEM allocator and MMA issuer (lane 0 issues; the whole warp
//                 clears the rows past a group's K in MN-major stages)
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31 and
//                 stores each 32 x 32 chunk row-contiguous through shared memory
// The accumulator is double-buffered in TMEM (2 x 256 fp32 columns), so the
// epilogue of one tile overlaps the main loop of the next.  Operands are
// K-major, or MN-major (B, and A with B) when K lies on the rows of the stored
// matrix: 64 x 64 TMA boxes and MN-major shared-memory descriptors.
//
// Every wait on an mbarrier is bounded (kWaitLimitNs); on expiry the kernel
// records MOE_ERR_TIMEOUT, every role leaves its loop, and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "tc_gemm.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;      // UMMA M (one CTA)
constexpr int kBK = 64;       // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kBN = 256;      // TMEM columns per accumulator buffer / max UMMA N
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1024;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kBBytes = kBN * kBK * 2;  // 32 KB
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * (kABytes + kBBytes) + 256;

struct KParams {
    int G;
    int64_t a_rows_per_group;
    int64_t b_rows_per_group;
    int64_t M;
    int64_t N;
    int n_tiles;
    int n_mma;        // UMMA N (multiple of 32, <= 256)
    int tile_n_out;   // output columns produced per tile
    int b_box_rows;   // rows per B TMA box (n_mma, or n_mma/2 for the dual form)
    int k_blocks;
    int k_split_blocks;  // MN-major B: K blocks from the first map before switching to the second (0: none)
    uint32_t tx_bytes;
    const int32_t* rows;
    const int32_t* k_rows;
    void* out;
    void* out2;       // rows m >= m_split of a group (0: none)
    int64_t m_split;
    const void* ab;   // SwiGLU backward: [a | b] beside the dh accumulator
    void* h_out;
    int64_t ldo;
    int64_t out_rows_per_group;
    const void* bias;
    int64_t bias_group_stride;
    int vec_ok;
    int tma_out;  // fp32 output through TMA stores (every tile row valid, N a multiple of 32)
    int32_t* status;
};

constexpr bool is_dual(int epi) { return epi == TC_EPI_SWIGLU || epi == TC_EPI_F32_DUAL; }

using namespace tc;

// Map a linear tile index to (group, m-tile, n-tile).  prefix[g] is the first
// tile of group g; tiles of a group run n fastest, so concurrently active CTAs
// share an m-tile of A and together write whole output rows (measured on B200:
// 33 us less per SwiGLU training step than m fastest, the forward unchanged; a
// group's operands stay in L2 either way).
__device__ __forceinline__ void decode_tile(int tile, const int* prefix, int G, int n_tiles, int& g,
                                            int& mt, int& nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    g = lo;
    const int local = tile - prefix[g];
    mt = local / n_tiles;
    nt = local - mt * n_tiles;
}

// K blocks of group g: all of them, or (k_rows given) those holding its first
// k_rows[g] K positions, at least one (the operands are zero past k_rows[g], so
// a group with none still produces its zero tile).
__device__ __forceinline__ int group_k_blocks(const KParams& p, int g) {
    if (p.k_rows == nullptr) return p.k_blocks;
    const int v = p.k_rows[g];
    const int kb = v <= 0 ? 1 : (v + kBK - 1) / kBK;
    return kb < p.k_blocks ? kb : p.k_blocks;
}

// Store 32 bf16 values (already packed in pairs) for columns n0..n0+31 of one row.
__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* row, int64_t n0, int64_t N, const uint32_t (&pk)[16],
                                              bool vec) {
    if (vec && n0 + 32 <= N) {
        uint4* dst = reinterpret_cast<uint4*>(row + n0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (n0 + i < N) {
                const uint32_t w = pk[i >> 1];
                const uint16_t h = (i & 1) ? (uint16_t)(w >> 16) : (uint16_t)(w & 0xFFFFu);
                row[n0 + i] = __ushort_as_bfloat16(h);
            }
        }
    }
}

// Drain n 32-column chunks of this thread's TMEM lane starting at t_row, with the
// load of chunk c + 1 in flight while chunk c is processed (its stores overlap the
// TMEM read latency).
template <typename F>
__device__ __forceinline__ void pipelined_chunks(uint32_t t_row, int n, F&& process) {
    uint32_t ra[32], rb[32];
    tmem_ld32(t_row, ra);
    tmem_ld_wait(ra);
    for (int c = 0; c < n; c += 2) {
        if (c + 1 < n) tmem_ld32(t_row + (c + 1) * 32, rb);
        process(c, ra);
        if (c + 1 < n) {
            tmem_ld_wait(rb);
            if (c + 2 < n) tmem_ld32(t_row + (c + 2) * 32, ra);
            process(c + 1, rb);
            if (c + 2 < n) tmem_ld_wait(ra);
        }
    }
}

template <int EPI, bool AMN, bool BMN>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut,
                   const __grid_constant__ CUtensorMap tmOut2, const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_prefix[kMaxGroups + 1];
    // epilogue staging, one 32 x 32 chunk per warp (1024-aligned: the TMA store reads it 128-byte swizzled)
    __shared__ __align__(1024) uint32_t s_stage[4][32 * 32];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smA = smem;
    uint8_t* smB = smem + kStages * kABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + kStages * kBBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = bars + 2 * kStages;
    uint64_t* tempty = bars + 2 * kStages + 2;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- setup: barriers, TMEM, tile table ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(2 * kBN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int g = threadIdx.x; g < p.G; g += blockDim.x) {
        int64_t r = p.rows ? (int64_t)p.rows[g] : p.M;
        r = r < 0 ? 0 : (r > p.M ? p.M : r);
        s_prefix[g + 1] = (int)((r + kBM - 1) / kBM);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        s_prefix[0] = 0;
        for (int g = 0; g < p.G; ++g) s_prefix[g + 1] = s_prefix[g] + s_prefix[g + 1] * p.n_tiles;
    }
    __syncthreads();
    const int total = s_prefix[p.G];
    const uint32_t tmem_base = s_tmem;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x) {
                int g, mt, nt;
                decode_tile(tile, s_prefix, p.G, p.n_tiles, g, mt, nt);
                const int32_t a_y = (int32_t)(g * p.a_rows_per_group + (int64_t)mt * kBM);
                const int32_t b_y = (int32_t)(g * p.b_rows_per_group + (int64_t)nt * p.b_box_rows);
                const int kbg = group_k_blocks(p, g);
                for (int kb = 0; kb < kbg; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&full[stage], p.tx_bytes);
                    uint8_t* a_dst = smA + stage * kABytes;
                    uint8_t* b_dst = smB + stage * kBBytes;
                    if (AMN) {
                        // K rows kb*64 .. +63 of the group's (K, M) matrix, two 64-column boxes of 8 KB
                        const int32_t k_y = (int32_t)(g * p.a_rows_per_group + (int64_t)kb * kBK);
                        tma_load_2d(a_dst, &tmA, mt * kBM, k_y, &full[stage]);
                        tma_load_2d(a_dst + 8192, &tmA, mt * kBM + 64, k_y, &full[stage]);
                    } else {
                        tma_load_2d(a_dst, &tmA, kb * kBK, a_y, &full[stage]);
                    }
                    if (BMN) {
                        // K rows kb*64 .. +63 of the (K, N) weight, in 64-column boxes of 8 KB
                        const bool second = p.k_split_blocks > 0 && kb >= p.k_split_blocks;
                        const int32_t k_y = (int32_t)(g * p.b_rows_per_group +
                                                      (int64_t)(kb - (second ? p.k_split_blocks : 0)) * kBK);
                        for (int i = 0; i < p.n_mma / 64; ++i)
                            tma_load_2d(b_dst + i * 8192, second ? &tmB2 : &tmB, nt * p.n_mma + 64 * i, k_y,
                                        &full[stage]);
                    } else {
                        tma_load_2d(b_dst, &tmB, kb * kBK, b_y, &full[stage]);
                    }
                    if (is_dual(EPI))
                        tma_load_2d(b_dst + p.b_box_rows * (kBK * 2), &tmB2, kb * kBK, b_y, &full[stage]);
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
        // Lane 0 issues the MMAs.  When the K range of a group ends inside a block
        // and an operand is MN-major (K on its rows), the whole warp first clears
        // that block's rows past the valid K in shared memory (they hold whatever
        // follows the group in memory), so garbage never meets a zero.
        constexpr bool kMask = AMN || BMN;
        const uint32_t idesc = make_idesc(kBM, p.n_mma) | (AMN ? (1u << 15) : 0u) | (BMN ? (1u << 16) : 0u);
        int stage = 0;
        uint32_t phase = 0;
        uint32_t it = 0;
        bool ready = false;  // lane 0: full[stage] was seen complete by an early test
        for (int tile = blockIdx.x;; tile += gridDim.x, ++it) {
            // one decision for the whole warp (s_abort may be raised by another warp meanwhile)
            if (!__shfl_sync(0xffffffffu, (tile < total && !s_abort) ? 1 : 0, 0)) break;
            const uint32_t acc = it & 1u;
            const uint32_t acc_phase = (it >> 1) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                s_abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * kBN;
            int g_, mt_, nt_;
            decode_tile(tile, s_prefix, p.G, p.n_tiles, g_, mt_, nt_);
            const int kbg = group_k_blocks(p, g_);
            int kvalid_last = kBK;  // valid K rows in the group's last block
            if (kMask && p.k_rows) {
                const int v = p.k_rows[g_];
                kvalid_last = v <= 0 ? 0 : v - (kbg - 1) * kBK;
                if (kvalid_last > kBK) kvalid_last = kBK;
            }
            for (int kb = 0; kb < kbg; ++kb) {
                // the group's last block: only the K steps of 16 that hold valid rows (at least one),
                // and only the rows between the last valid one and the end of those steps are cleared
                const bool last = kMask && kb == kbg - 1 && kvalid_last < kBK;
                const int nkk = last ? (kvalid_last <= 0 ? 1 : (kvalid_last + 15) / 16) : kBK / 16;
                const int kend = nkk * 16;
                const bool clear = last && kvalid_last < kend;
                int okf = 1;
                if ((lane == 0 && !ready) || (lane != 0 && clear)) okf = mbar_wait(&full[stage], phase, p.status) ? 1 : 0;
                okf = __all_sync(0xffffffffu, okf);
                if (!okf) {
                    s_abort = 1;
                    ok = 0;
                    break;
                }
                if (clear) {
                    // rows [kvalid_last, kend) of every 8 KB MN-major box: 128 bytes per row
                    const int nrow = kend - (kvalid_last < 0 ? 0 : kvalid_last);
                    const int r0 = kend - nrow;
                    if (AMN) {
                        uint8_t* base = smA + stage * kABytes;
                        for (int i = lane; i < 2 * nrow * 8; i += 32) {
                            const int box = i / (nrow * 8), rem = i - box * nrow * 8;
                            *reinterpret_cast<uint4*>(base + box * 8192 + (r0 + rem / 8) * 128 + (rem & 7) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    if (BMN) {
                        uint8_t* base = smB + stage * kBBytes;
                        const int nbox = p.n_mma / 64;
                        for (int i = lane; i < nbox * nrow * 8; i += 32) {
                            const int box = i / (nrow * 8), rem = i - box * nrow * 8;
                            *reinterpret_cast<uint4*>(base + box * 8192 + (r0 + rem / 8) * 128 + (rem & 7) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) {
                    tc_fence_after();
                    const uint64_t ad = AMN ? sw128_mn_desc(smem_u32(smA + stage * kABytes), 8192)
                                            : sw128_desc(smem_u32(smA + stage * kABytes));
                    const uint64_t bd = BMN ? sw128_mn_desc(smem_u32(smB + stage * kBBytes), 8192)
                                            : sw128_desc(smem_u32(smB + stage * kBBytes));
                    // a K step of 16: 32 bytes along a K-major row, or two 1024-byte groups of 8 K rows
                    const int ns = stage + 1 == kStages ? 0 : stage + 1;
                    const uint32_t np = stage + 1 == kStages ? phase ^ 1u : phase;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        if (kk < nkk)
                            tc_mma(d_tmem, ad + (AMN ? 128 : 2) * kk, bd + (BMN ? 128 : 2) * kk, idesc,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
                        // the tensor core takes new MMAs only as it finishes old ones: look at the
                        // next stage while this one's MMAs are being accepted
                        if (kk == 1) ready = mbar_test(smem_u32(&full[ns]), np);
                    }
                    tc_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&tfull[acc]);
            __syncwarp();
        }
    } else {
        // -------------------------------- epilogue --------------------------------
        const int q = warp & 3;
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int g, mt, nt;
            decode_tile(tile, s_prefix, p.G, p.n_tiles, g, mt, nt);
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
            const int row = q * 32 + lane;
            const int64_t m = (int64_t)mt * kBM + row;
            int64_t rows_g = p.rows ? (int64_t)p.rows[g] : p.M;
            rows_g = rows_g > p.M ? p.M : rows_g;
            const bool row_ok = m < rows_g;
            // the m-tiles past m_split write the second output (a tile lies wholly on one side)
            const bool second = p.m_split > 0 && (int64_t)mt * kBM >= p.m_split;
            void* const outp = second ? p.out2 : p.out;
            const int64_t out_row = (int64_t)g * p.out_rows_per_group + m - (second ? p.m_split : 0);
            const uint32_t t_row = tmem_base + acc * kBN + ((uint32_t)(q * 32) << 16);
            // this warp's 32 rows for the staged stores
            const int64_t wrow0 = (int64_t)mt * kBM + q * 32;
            const int wrows = (int)(rows_g - wrow0 < 0 ? 0 : (rows_g - wrow0 > 32 ? 32 : rows_g - wrow0));
            const int64_t out_wrow0 = (int64_t)g * p.out_rows_per_group + wrow0 - (second ? p.m_split : 0);
            uint32_t* stg = s_stage[q];

            if (EPI == TC_EPI_SWIGLU) {
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(outp) + out_row * p.ldo;
                const int half = p.n_mma / 2;
                for (int c = 0; c < half / 32; ++c) {
                    uint32_t rg[32], ru[32];
                    tmem_ld32(t_row + c * 32, rg);
                    tmem_ld_wait(rg);
                    tmem_ld32(t_row + half + c * 32, ru);
                    tmem_ld_wait(ru);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float h0 = silu_f(__uint_as_float(rg[2 * i])) * __uint_as_float(ru[2 * i]);
                        const float h1 = silu_f(__uint_as_float(rg[2 * i + 1])) * __uint_as_float(ru[2 * i + 1]);
                        pk[i] = pack_bf16x2(h0, h1);
                    }
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + c * 32;
                    if (p.vec_ok && n0 + 32 <= p.N)
                        warp_store_chunk<16>(stg, pk,
                                             reinterpret_cast<uint8_t*>(reinterpret_cast<__nv_bfloat16*>(outp) +
                                                                        out_wrow0 * p.ldo + n0),
                                             p.ldo * 2, wrows, lane);
                    else if (row_ok)
                        store_bf16_32(orow, n0, p.N, pk, p.vec_ok);
                }
            } else if (EPI == TC_EPI_SWIGLU_BWD) {
                // acc = dh.  With s = sigmoid(a): h = a s b, da = dh b (s + a s (1 - s)), db = dh a s.
                // The warp's 32 rows x 32 columns of [a | b] for a chunk arrive as coalesced loads (one
                // row's 64 + 64 bytes per 8 lanes), issued two chunks ahead of the math and turned
                // row-per-lane through the staging buffer; the three bf16 results leave through the
                // staged coalesced stores.  (An L2 prefetch of the tile by the producer measured slower.)
                // The sigmoid takes the fast reciprocal (2 ulp): the correctly rounded one cost the
                // epilogue more than the whole of its loads.
                const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(p.ab);
                __nv_bfloat16* hb = reinterpret_cast<__nv_bfloat16*>(p.h_out);
                __nv_bfloat16* dab = reinterpret_cast<__nv_bfloat16*>(outp);
                const int nch = p.n_mma / 32;  // even: n_mma is a multiple of 64 with an MN-major B
                const int lr = lane >> 3, piece = lane & 7;
                auto load_ab = [&](const int c, uint4 (&v)[8]) {
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + c * 32;
                    const int64_t col = (piece < 4 ? n0 : p.N + n0) + 8 * (piece & 3);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = lr + 4 * i;
                        v[i] = (r < wrows && n0 < p.N)
                                   ? __ldg(reinterpret_cast<const uint4*>(ab + (out_wrow0 + r) * p.ldo + col))
                                   : make_uint4(0u, 0u, 0u, 0u);
                    }
                };
                auto chunk = [&](const int c, uint4 (&v)[8]) {
                    uint32_t r[32];
                    tmem_ld32(t_row + c * 32, r);
                    // rows to lanes: row lr + 4i, 16-byte piece `piece` (a: 0-3, b: 4-7)
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = lr + 4 * i;
                        *reinterpret_cast<uint4*>(stg + rr * 32 + 4 * (piece ^ (rr & 7))) = v[i];
                    }
                    __syncwarp();
                    uint32_t aw[16], bw[16];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint4 q4 = *reinterpret_cast<const uint4*>(stg + lane * 32 + 4 * (k ^ (lane & 7)));
                        uint32_t* d = k < 4 ? aw + 4 * k : bw + 4 * (k - 4);
                        d[0] = q4.x, d[1] = q4.y, d[2] = q4.z, d[3] = q4.w;
                    }
                    __syncwarp();
                    if (c + 2 < nch) load_ab(c + 2, v);
                    tmem_ld_wait(r);
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + c * 32;
                    if (n0 < p.N) {
                        uint32_t ph[16], pa[16], pb[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float hv[2], dav[2], dbv[2];
#pragma unroll
                            for (int m2 = 0; m2 < 2; ++m2) {
                                const float a = __uint_as_float(m2 ? (aw[i] & 0xFFFF0000u) : (aw[i] << 16));
                                const float b = __uint_as_float(m2 ? (bw[i] & 0xFFFF0000u) : (bw[i] << 16));
                                const float gd = __uint_as_float(r[2 * i + m2]);
                                const float sg = __fdividef(1.0f, 1.0f + __expf(-a));
                                const float as = a * sg;
                                hv[m2] = as * b;
                                dbv[m2] = gd * as;
                                dav[m2] = (gd * b) * fmaf(as, 1.0f - sg, sg);
                            }
                            ph[i] = pack_bf16x2(hv[0], hv[1]);
                            pa[i] = pack_bf16x2(dav[0], dav[1]);
                            pb[i] = pack_bf16x2(dbv[0], dbv[1]);
                        }
                        warp_store_chunk<16>(stg, ph, reinterpret_cast<uint8_t*>(hb + out_wrow0 * p.N + n0), p.N * 2,
                                             wrows, lane);
                        warp_store_chunk<16>(stg, pa, reinterpret_cast<uint8_t*>(dab + out_wrow0 * p.ldo + n0),
                                             p.ldo * 2, wrows, lane);
                        warp_store_chunk<16>(stg, pb,
                                             reinterpret_cast<uint8_t*>(dab + out_wrow0 * p.ldo + p.N + n0),
                                             p.ldo * 2, wrows, lane);
                    }
                };
                uint4 v0[8], v1[8];
                load_ab(0, v0);
                load_ab(1, v1);
#pragma unroll 1
                for (int c = 0; c < nch; c += 2) {
                    chunk(c, v0);
                    chunk(c + 1, v1);
                }
            } else if (EPI == TC_EPI_F32_DUAL) {
                // gate half of the accumulator -> columns [0, N), up half -> [N, 2N)
                float* orow = reinterpret_cast<float*>(outp) + out_row * p.ldo;
                const int half = p.n_mma / 2;
                for (int c = 0; c < p.n_mma / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(t_row + c * 32, r);
                    tmem_ld_wait(r);
                    const bool up = c * 32 >= half;
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + (up ? c * 32 - half : c * 32);
                    float* dst = orow + (up ? p.N : 0);
                    if (p.vec_ok && n0 + 32 <= p.N) {
                        warp_store_chunk<32>(stg, r,
                                             reinterpret_cast<uint8_t*>(reinterpret_cast<float*>(outp) +
                                                                        out_wrow0 * p.ldo + (up ? p.N : 0) + n0),
                                             p.ldo * 4, wrows, lane);
                    } else if (row_ok) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (n0 + i < p.N) dst[n0 + i] = __uint_as_float(r[i]);
                    }
                }
            } else if (EPI == TC_EPI_F32 && AMN && BMN && p.tma_out) {
                // the weight-gradient form: every row valid, full 32-column chunks.  Each chunk goes
                // to the warp's staging buffer in the map's 128-byte swizzled layout (conflict-free:
                // lane = row) and one lane hands it to the TMA, which streams it out while the warp
                // drains the next chunk; the buffer is rewritten only once the TMA has read it.
                auto process = [&](const int c, const uint32_t (&r)[32]) {
                    if ((int64_t)nt * p.tile_n_out + c * 32 >= p.N) return;  // past N (warp-uniform)
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
#pragma unroll
                    for (int m = 0; m < 8; ++m)
                        *reinterpret_cast<uint4*>(stg + lane * 32 + 4 * (m ^ (lane & 7))) =
                            make_uint4(r[4 * m], r[4 * m + 1], r[4 * m + 2], r[4 * m + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(second ? &tmOut2 : &tmOut, stg, (int32_t)(nt * p.tile_n_out + c * 32), (int32_t)out_wrow0);
                        bulk_commit();
                    }
                };
                pipelined_chunks(t_row, p.n_mma / 32, process);
            } else if (EPI == TC_EPI_F32) {
                float* orow = reinterpret_cast<float*>(outp) + out_row * p.ldo;
                const float* bias = reinterpret_cast<const float*>(p.bias);
                auto process = [&](const int c, const uint32_t (&r)[32]) {
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + c * 32;
                    if (p.vec_ok && n0 + 32 <= p.N) {
                        uint32_t w[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            w[i] = __float_as_uint(__uint_as_float(r[i]) + (bias ? bias[n0 + i] : 0.f));
                        warp_store_chunk<32>(stg, w,
                                             reinterpret_cast<uint8_t*>(reinterpret_cast<float*>(outp) +
                                                                        out_wrow0 * p.ldo + n0),
                                             p.ldo * 4, wrows, lane);
                    } else if (row_ok) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (n0 + i < p.N) orow[n0 + i] = __uint_as_float(r[i]) + (bias ? bias[n0 + i] : 0.f);
                    }
                };
                pipelined_chunks(t_row, p.n_mma / 32, process);
            } else {
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(outp) + out_row * p.ldo;
                const __nv_bfloat16* bias =
                    reinterpret_cast<const __nv_bfloat16*>(p.bias) + (p.bias ? g * p.bias_group_stride : 0);
                auto process = [&](const int c, const uint32_t (&r)[32]) {
                    const int64_t n0 = (int64_t)nt * p.tile_n_out + c * 32;
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float v0 = __uint_as_float(r[2 * i]);
                        float v1 = __uint_as_float(r[2 * i + 1]);
                        if (EPI == TC_EPI_BF16_BIAS || EPI == TC_EPI_GELU_BIAS) {
                            const int64_t na = n0 + 2 * i, nb = n0 + 2 * i + 1;
                            v0 += na < p.N ? __bfloat162float(bias[na]) : 0.f;
                            v1 += nb < p.N ? __bfloat162float(bias[nb]) : 0.f;
                        }
                        if (EPI == TC_EPI_GELU_BIAS) {
                            v0 = gelu_f(v0);
                            v1 = gelu_f(v1);
                        }
                        pk[i] = pack_bf16x2(v0, v1);
                    }
                    if (p.vec_ok && n0 + 32 <= p.N)
                        warp_store_chunk<16>(stg, pk,
                                             reinterpret_cast<uint8_t*>(reinterpret_cast<__nv_bfloat16*>(outp) +
                                                                        out_wrow0 * p.ldo + n0),
                                             p.ldo * 2, wrows, lane);
                    else if (row_ok)
                        store_bf16_32(orow, n0, p.N, pk, p.vec_ok);
                };
                pipelined_chunks(t_row, p.n_mma / 32, process);
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (s_abort) break;
        }
        if (EPI == TC_EPI_F32 && AMN && BMN && p.tma_out && lane == 0) bulk_wait_all();  // stores done before exit
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kBN)
                     : "memory");
    }
}

// ------------------------------- host side ---------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

// 2-D bf16 map over a (rows, inner) row-major matrix, box = (box_rows, 64),
// 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld_elems * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D fp32 map over a (rows, inner) row-major matrix: box = box_rows x 32
// elements (128 bytes), 128-byte swizzle, zero fill outside the matrix.
bool make_map_f32(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld_elems * 4};
    cuuint32_t box[2] = {32u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D fp32 map read MN-major by the tf32 MMA: box = box_rows x 32 elements (128
// bytes), 128-byte swizzle of 32-byte chunks (the layout tf32 MN-major operands take).
bool make_map_f32_mn(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld_elems, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld_elems * 4};
    cuuint32_t box[2] = {32u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

template <int EPI, bool AMN = false, bool BMN = false>
int launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const CUtensorMap& out,
           const CUtensorMap& out2, const KParams& kp, int grid, cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(tc_gemm_kernel<EPI, AMN, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kSmemBytes));
        attr_set[dev] = true;
    }
    tc_gemm_kernel<EPI, AMN, BMN><<<grid, kThreads, kSmemBytes, stream>>>(a, b, b2, out, out2, kp);
    return launch_status();
}

}  // namespace

int tc_gemm_run(const TcGemmProblem& p, cudaStream_t stream) {
    MOE_REQUIRE(p.a && p.b && p.out, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G >= 1 && p.M >= 1 && p.N >= 1 && p.K >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(p.G <= kMaxGroups, MOE_ERR_UNSUPPORTED);
    // TMA: 16-byte aligned bases, row strides a multiple of 16 bytes.
    MOE_REQUIRE(aligned16(p.a) && aligned16(p.b) && (p.lda * 2) % 16 == 0 && (p.ldb * 2) % 16 == 0,
                MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE((p.a_mn_major ? p.lda >= p.M : p.lda >= p.K) && (p.b_mn_major ? p.ldb >= p.N : p.ldb >= p.K),
                MOE_ERR_INVALID_ARG);
    // MN-major A is built for the weight-gradient products: fp32 out, MN-major B, K rows per group
    if (p.a_mn_major)
        MOE_REQUIRE(p.b_mn_major && p.epilogue == TC_EPI_F32 && p.k_split == 0 && p.rows == nullptr,
                    MOE_ERR_UNSUPPORTED);
    // the split output: MN-major A only, whole m-tiles on each side
    MOE_REQUIRE(p.m_split >= 0, MOE_ERR_INVALID_ARG);
    if (p.m_split > 0)
        MOE_REQUIRE(p.a_mn_major && p.out2 && p.m_split % kBM == 0 && p.m_split < p.M &&
                        p.out_rows_per_group >= p.m_split && p.out_rows_per_group >= p.M - p.m_split,
                    MOE_ERR_INVALID_ARG);
    if (p.b_mn_major) {
        MOE_REQUIRE(p.epilogue == TC_EPI_F32 || p.epilogue == TC_EPI_BF16 || p.epilogue == TC_EPI_SWIGLU_BWD,
                    MOE_ERR_UNSUPPORTED);
        MOE_REQUIRE(p.k_split % kBK == 0 && p.k_split >= 0 && p.k_split < p.K, MOE_ERR_UNSUPPORTED);
        MOE_REQUIRE(p.k_split == 0 || (p.b2 && aligned16(p.b2)), MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(p.b_rows_per_group >= (p.k_split > 0 ? p.k_split : p.K), MOE_ERR_INVALID_ARG);
    }
    // the SwiGLU backward epilogue: MN-major B, whole 32-column chunks, 16-byte aligned rows
    if (p.epilogue == TC_EPI_SWIGLU_BWD)
        MOE_REQUIRE(p.b_mn_major && !p.a_mn_major && p.ab && p.h && aligned16(p.ab) && aligned16(p.h) &&
                        p.N % 32 == 0 && p.ldo >= 2 * p.N && p.m_split == 0,
                    MOE_ERR_UNSUPPORTED);
    const bool dual = p.epilogue == TC_EPI_SWIGLU || p.epilogue == TC_EPI_F32_DUAL;
    if (dual) MOE_REQUIRE(p.b2 && aligned16(p.b2), MOE_ERR_INVALID_ARG);
    // TMA coordinates are 32-bit.
    MOE_REQUIRE(p.a_rows_total < (int64_t(1) << 31) && p.b_rows_total < (int64_t(1) << 31), MOE_ERR_UNSUPPORTED);

    KParams kp{};
    kp.G = p.G;
    kp.a_rows_per_group = p.a_rows_per_group;
    kp.b_rows_per_group = p.b_rows_per_group;
    kp.M = p.M;
    kp.N = p.N;
    if (dual) {
        kp.n_mma = kBN;
        kp.tile_n_out = kBN / 2;
        kp.b_box_rows = kBN / 2;
    } else {
        int64_t n = (p.N + 31) / 32 * 32;
        kp.n_mma = (int)(n < kBN ? n : kBN);
        kp.tile_n_out = kp.n_mma;
        kp.b_box_rows = kp.n_mma;
    }
    if (p.b_mn_major) MOE_REQUIRE(kp.n_mma % 64 == 0, MOE_ERR_UNSUPPORTED);
    kp.n_tiles = (int)((p.N + kp.tile_n_out - 1) / kp.tile_n_out);
    kp.k_blocks = (int)((p.K + kBK - 1) / kBK);
    kp.k_split_blocks = p.b_mn_major ? (int)(p.k_split / kBK) : 0;
    kp.tx_bytes = (uint32_t)(kABytes + kp.n_mma * kBK * 2);
    kp.rows = p.rows;
    kp.k_rows = p.k_rows;
    kp.out = p.out;
    kp.out2 = p.m_split > 0 ? p.out2 : nullptr;
    kp.m_split = p.m_split;
    kp.ab = p.ab;
    kp.h_out = p.h;
    kp.ldo = p.ldo;
    kp.out_rows_per_group = p.out_rows_per_group;
    kp.bias = p.bias;
    kp.bias_group_stride = p.bias_group_stride;
    const bool f32_out = p.epilogue == TC_EPI_F32 || p.epilogue == TC_EPI_F32_DUAL;
    const size_t esz = f32_out ? 4 : 2;
    kp.vec_ok = aligned16(p.out) && (p.ldo * (int64_t)esz) % 16 == 0 && (p.m_split == 0 || aligned16(p.out2));
    if (p.epilogue == TC_EPI_F32_DUAL) kp.vec_ok = kp.vec_ok && (p.N * 4) % 16 == 0;
    if (p.epilogue == TC_EPI_SWIGLU_BWD) MOE_REQUIRE(kp.vec_ok, MOE_ERR_UNSUPPORTED);
    kp.status = p.status;
    // the weight-gradient form writes whole 32 x 32 fp32 boxes through the TMA
    kp.tma_out = p.a_mn_major && p.epilogue == TC_EPI_F32 && p.rows == nullptr && p.bias == nullptr &&
                 p.M % kBM == 0 && p.N % 32 == 0 && kp.vec_ok &&
                 (p.m_split > 0 || p.out_rows_per_group >= p.M) &&
                 (int64_t)p.G * p.out_rows_per_group < (int64_t(1) << 31);

    CUtensorMap ma, mb, mb2, mo, mo2;
    if (p.a_mn_major)  // (K rows, M columns) with 64 x 64 boxes
        MOE_REQUIRE(make_map(&ma, p.a, p.M, p.a_rows_total, p.lda, kBK), MOE_ERR_CUDA);
    else
        MOE_REQUIRE(make_map(&ma, p.a, p.K, p.a_rows_total, p.lda, kBM), MOE_ERR_CUDA);
    if (p.b_mn_major) {
        // (K rows, N columns) with 64 x 64 boxes: rows past b_rows_total and columns past N read as zero
        MOE_REQUIRE(make_map(&mb, p.b, p.N, p.b_rows_total, p.ldb, kBK), MOE_ERR_CUDA);
        if (p.k_split > 0) MOE_REQUIRE(make_map(&mb2, p.b2, p.N, p.b_rows_total, p.ldb, kBK), MOE_ERR_CUDA);
        else mb2 = mb;
    } else {
        MOE_REQUIRE(make_map(&mb, p.b, p.K, p.b_rows_total, p.ldb, kp.b_box_rows), MOE_ERR_CUDA);
        if (dual) MOE_REQUIRE(make_map(&mb2, p.b2, p.K, p.b_rows_total, p.ldb, kp.b_box_rows), MOE_ERR_CUDA);
        else mb2 = mb;
    }

    const int64_t max_tiles = (int64_t)p.G * ((p.M + kBM - 1) / kBM) * kp.n_tiles;
    MOE_REQUIRE(max_tiles < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    int grid = device_sm_count();
    if (max_tiles < grid) grid = (int)max_tiles;
    if (grid < 1) grid = 1;

    if (kp.tma_out)
        MOE_REQUIRE(make_map_f32(&mo, p.out, p.N, (int64_t)p.G * p.out_rows_per_group, p.ldo, 32), MOE_ERR_CUDA);
    else
        mo = ma;  // unused
    if (kp.tma_out && p.m_split > 0)
        MOE_REQUIRE(make_map_f32(&mo2, p.out2, p.N, (int64_t)p.G * p.out_rows_per_group, p.ldo, 32), MOE_ERR_CUDA);
    else
        mo2 = mo;  // unused
    if (p.a_mn_major) return launch<TC_EPI_F32, true, true>(ma, mb, mb2, mo, mo2, kp, grid, stream);
    if (p.b_mn_major) {
        if (p.epilogue == TC_EPI_SWIGLU_BWD)
            return launch<TC_EPI_SWIGLU_BWD, false, true>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        return p.epilogue == TC_EPI_F32 ? launch<TC_EPI_F32, false, true>(ma, mb, mb2, mo, mo2, kp, grid, stream)
                                        : launch<TC_EPI_BF16, false, true>(ma, mb, mb2, mo, mo2, kp, grid, stream);
    }
    switch (p.epilogue) {
        case TC_EPI_F32: return launch<TC_EPI_F32>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        case TC_EPI_BF16: return launch<TC_EPI_BF16>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        case TC_EPI_BF16_BIAS: return launch<TC_EPI_BF16_BIAS>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        case TC_EPI_GELU_BIAS: return launch<TC_EPI_GELU_BIAS>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        case TC_EPI_SWIGLU: return launch<TC_EPI_SWIGLU>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        case TC_EPI_F32_DUAL: return launch<TC_EPI_F32_DUAL>(ma, mb, mb2, mo, mo2, kp, grid, stream);
        default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace moe
