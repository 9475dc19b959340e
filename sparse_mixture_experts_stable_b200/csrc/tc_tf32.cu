// fp32 grouped GEMM as split-tf32 products on sm_100a (see tc_tf32.cuh).
//
// An operand that is already fp32 and K-major in memory (a_trans false / b_trans
// true, contiguous groups, no per-group K limit) is not split beforehand: the
// TMA brings its raw fp32 tile into the stage's "hi" slot and four converter
// warps write lo = x - trunc(x) into the "lo" slot.  The tf32 MMA reads a raw
// fp32 operand as its value truncated to tf32 (its low 13 mantissa bits
// ignored; checked on the hardware), so the raw tile is exactly the hi part
// and lo is exact in fp32.  (With truncation |lo| < 2^-10 |x|, so the dropped
// lo*lo product stays below 2^-20 |a*b|.)  Other operands go through:
// 1. split_kernel writes hi/lo of A as (G, M, Kp) and of B as (G, N, Kp),
//    K-major, Kp = K rounded up to 32 (one 128-byte swizzle row of fp32), with
//    zeros for k >= the group's valid K; transposed source forms go through a
//    32 x 32 shared-memory tile so both the reads and the writes are coalesced.
// 2. tf32x3_kernel: persistent, one CTA of 192 threads per SM.  Warp 0 issues
//    TMA loads of the four operand tiles (A hi/lo: 128 rows, B hi/lo: up to 128
//    rows, 32 K each) into a 3-stage ring; warp 1 owns TMEM (2 x 128 fp32
//    columns, double-buffered) and issues, per K step of 8, three
//    tcgen05.mma.kind::tf32 into one accumulator; warps 2..5 read TMEM and apply
//    the epilogue.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "tc_gemm.cuh"
#include "tc_ptx.cuh"
#include "tc_tf32.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kBM = 128;                 // rows of A per tile (UMMA M)
constexpr int kBN = 128;                 // max rows of B per tile (UMMA N)
constexpr int kBK = 32;                  // fp32 elements per 128-byte swizzle row
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kConvThreads = 128;  // converter warps for raw operands (after the 192 threads above)
// MN-major raw operands: TMA-loaded with the 128-byte swizzle on a 32-byte base, the layout
// the tf32 MMA reads with its transpose bits (layout type 1 in the shared-memory descriptor).
constexpr bool kRawMnMajor = true;
constexpr int kMaxGroups = 1024;
constexpr int kTileBytes = 128 * kBK * 4;   // 16 KB per operand tile
constexpr int kStageBytes = 4 * kTileBytes;  // A hi, A lo, B hi, B lo
constexpr int kAccCols = 128;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

__device__ __forceinline__ float tf32_round(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// out[g][r][k] (k < Kp) = hi/lo of src(g, r, k) for k < valid K, else 0.
//   TRANS: src(g, r, k) = src[g*gs + k*ld + r]   (r contiguous in memory)
//   else : src(g, r, k) = src[g*gs + r*ld + k]   (k contiguous)
// Block 32 x 8 threads covers 32 rows x 32 k; grid (Kp/32, ceil(R/32), G).
template <bool TRANS, typename In>
__global__ void __launch_bounds__(256)
    split_kernel(const In* __restrict__ src, int64_t ld, int64_t gs, int64_t R, int64_t K, int64_t Kp,
                 const int32_t* __restrict__ krows, float* __restrict__ hi, float* __restrict__ lo) {
    __shared__ float tile[32][33];
    const int g = blockIdx.z;
    int64_t Kg = K;
    if (krows) {
        const int64_t r = krows[g];
        Kg = r < 0 ? 0 : (r < K ? r : K);
    }
    const int64_t r0 = (int64_t)blockIdx.y * 32, k0 = (int64_t)blockIdx.x * 32;
    const In* s = src + g * gs;
    const int tx = threadIdx.x, ty = threadIdx.y;
    if (TRANS) {
        // read 32 k-rows of 32 consecutive r, write transposed
        for (int i = ty; i < 32; i += 8) {
            const int64_t k = k0 + i, r = r0 + tx;
            tile[i][tx] = (k < Kg && r < R) ? to_f32(s[k * ld + r]) : 0.f;
        }
        __syncthreads();
        for (int i = ty; i < 32; i += 8) {
            const int64_t r = r0 + i, k = k0 + tx;
            if (r < R) {
                const float x = tile[tx][i];
                const float h = tf32_round(x);
                const size_t o = ((size_t)g * R + r) * Kp + k;
                hi[o] = h;
                lo[o] = x - h;
            }
        }
    } else {
        for (int i = ty; i < 32; i += 8) {
            const int64_t r = r0 + i, k = k0 + tx;
            if (r < R) {
                const float x = k < Kg ? to_f32(s[r * ld + k]) : 0.f;
                const float h = tf32_round(x);
                const size_t o = ((size_t)g * R + r) * Kp + k;
                hi[o] = h;
                lo[o] = x - h;
            }
        }
    }
}

struct T3Params {
    int G;
    int64_t M, N;
    int n_tiles;
    int n_mma;
    int k_blocks;
    uint32_t tx_bytes;
    int a_raw;  // A's hi slot holds the raw fp32 tile; the converter warps write its lo slot
    int b_raw;
    int a_mn;   // the raw tile is MN-major (4 KB atoms of 32 K rows x 32 fp32 along M or N)
    int b_mn;
    int64_t a_rows_per_group;  // MN-major raw operands: rows (K positions) of a group in memory
    int64_t b_rows_per_group;
    const int32_t* krows;      // per-group valid K (rows past it are zeroed in the stage), or NULL
    int64_t K;
    const int32_t* rows;
    int rows_mode;
    float* C;
    int64_t ldc;
    int64_t c_group_stride;
    const float* bias;
    int64_t bias_group_stride;
    int epilogue;
    int vec_ok;  // C, ldc (and bias, bias_group_stride) allow 16-byte accesses
    int tma_out; // plain fp32 out, every tile row valid: 32 x 32 chunks leave through TMA stores (tmC)
    int32_t* status;
};

// kind::tf32 instruction descriptor: D fp32, A and B tf32, both K-major.
__device__ __forceinline__ uint32_t make_idesc_tf32(int m, int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ int64_t group_m(const T3Params& p, int g) {
    if (p.rows_mode != 1) return p.M;
    const int64_t r = p.rows[g];
    return r < 0 ? 0 : (r < p.M ? r : p.M);
}

__device__ __forceinline__ void decode_tile(int tile, const int* prefix, int G, int n_tiles, int& g, int& mt,
                                            int& nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    g = lo;
    const int local = tile - prefix[g];
    // n fastest: concurrently active CTAs share an m-tile of A and write whole output rows
    // (measured on B200: the fp32 fwd+bwd step 5 us shorter than with m fastest)
    mt = local / n_tiles;
    nt = local - mt * n_tiles;
}

__global__ void __launch_bounds__(kThreads + kConvThreads, 1)
    tf32x3_kernel(const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
                  const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmBl,
                  const __grid_constant__ CUtensorMap tmC, const T3Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_prefix[kMaxGroups + 1];
    // epilogue staging, one 32 x 32 chunk per warp (1024-aligned: a TMA store reads it 128-byte swizzled)
    __shared__ __align__(1024) uint32_t s_stage[4][32 * 32];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = bars + 2 * kStages;
    uint64_t* tempty = bars + 2 * kStages + 2;
    uint64_t* conv = bars + 2 * kStages + 4;  // the converter warps have written the stage's lo slots
    const bool any_raw = p.a_raw || p.b_raw;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&conv[s], kConvThreads);
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
    for (int g = threadIdx.x; g < p.G; g += blockDim.x)
        s_prefix[g + 1] = (int)((group_m(p, g) + kBM - 1) / kBM) * p.n_tiles;
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
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x) {
                int g, mt, nt;
                decode_tile(tile, s_prefix, p.G, p.n_tiles, g, mt, nt);
                const int32_t a_y = (int32_t)(g * p.M + (int64_t)mt * kBM);
                const int32_t b_y = (int32_t)(g * p.N + (int64_t)nt * p.n_mma);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&full[stage], p.tx_bytes);
                    uint8_t* st = smem + stage * kStageBytes;
                    if (p.a_mn) {  // four 32 x 32 atoms along M
                        const int32_t ky = (int32_t)(g * p.a_rows_per_group + (int64_t)kb * kBK);
                        for (int i = 0; i < kBM / 32; ++i)
                            tma_load_2d(st + i * 4096, &tmAh, mt * kBM + 32 * i, ky, &full[stage]);
                    } else {
                        tma_load_2d(st, &tmAh, kb * kBK, a_y, &full[stage]);
                        if (!p.a_raw) tma_load_2d(st + kTileBytes, &tmAl, kb * kBK, a_y, &full[stage]);
                    }
                    if (p.b_mn) {
                        const int32_t ky = (int32_t)(g * p.b_rows_per_group + (int64_t)kb * kBK);
                        for (int i = 0; i < p.n_mma / 32; ++i)
                            tma_load_2d(st + 2 * kTileBytes + i * 4096, &tmBh, nt * p.n_mma + 32 * i, ky,
                                        &full[stage]);
                    } else {
                        tma_load_2d(st + 2 * kTileBytes, &tmBh, kb * kBK, b_y, &full[stage]);
                        if (!p.b_raw) tma_load_2d(st + 3 * kTileBytes, &tmBl, kb * kBK, b_y, &full[stage]);
                    }
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
            const uint32_t idesc =
                make_idesc_tf32(kBM, p.n_mma) | (p.a_mn ? (1u << 15) : 0u) | (p.b_mn ? (1u << 16) : 0u);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t it = 0;
            bool ready = false;  // the next stage was seen complete by an early test
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x, ++it) {
                const uint32_t acc = it & 1u;
                const uint32_t acc_phase = (it >> 1) & 1u;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ready && !mbar_wait(any_raw ? &conv[stage] : &full[stage], phase, p.status)) {
                        s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + stage * kStageBytes);
                    // K-major: a K step of 8 is 32 bytes along the row (2 descriptor units); MN-major:
                    // 8 K rows of 128 bytes (64 units), atoms 4 KB apart
                    const uint64_t ah = p.a_mn ? sw128b32_mn_desc(st, 4096) : sw128_desc(st);
                    const uint64_t al = p.a_mn ? sw128b32_mn_desc(st + kTileBytes, 4096) : sw128_desc(st + kTileBytes);
                    const uint64_t bh =
                        p.b_mn ? sw128b32_mn_desc(st + 2 * kTileBytes, 4096) : sw128_desc(st + 2 * kTileBytes);
                    const uint64_t bl =
                        p.b_mn ? sw128b32_mn_desc(st + 3 * kTileBytes, 4096) : sw128_desc(st + 3 * kTileBytes);
                    const uint32_t sa = p.a_mn ? 64u : 2u, sb = p.b_mn ? 64u : 2u;
                    const int ns = stage + 1 == kStages ? 0 : stage + 1;
                    const uint32_t np = stage + 1 == kStages ? phase ^ 1u : phase;
#pragma unroll
                    for (int ks = 0; ks < kBK / 8; ++ks) {
                        const uint32_t first = (kb == 0 && ks == 0) ? 0u : 1u;
                        mma_tf32(d_tmem, al + sa * ks, bh + sb * ks, idesc, first);
                        mma_tf32(d_tmem, ah + sa * ks, bl + sb * ks, idesc, 1u);
                        mma_tf32(d_tmem, ah + sa * ks, bh + sb * ks, idesc, 1u);
                        // the tensor core takes new MMAs only as it finishes old ones: look at the
                        // next stage while this one's MMAs are being accepted
                        if (ks == 1) ready = mbar_test(smem_u32(any_raw ? &conv[ns] : &full[ns]), np);
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
    } else if (warp >= kThreads / 32) {
        // -------------------------- raw-operand converters --------------------------
        // For each stage: lo = x - trunc(x) of every raw fp32 tile element, written
        // at the same position of the lo slot (the swizzled layout is elementwise).
        if (any_raw) {
            const int ct = threadIdx.x - kThreads;
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x) {
                int g, mt_, nt_;
                decode_tile(tile, s_prefix, p.G, p.n_tiles, g, mt_, nt_);
                int64_t kv = p.krows ? (int64_t)p.krows[g] : p.K;  // MN-major rows past it read the next group
                if (kv > p.K) kv = p.K;
                const int kval = (int)kv;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    int ok = 1;
                    if (lane == 0) ok = mbar_wait(&full[stage], phase, p.status) ? 1 : 0;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) {
                        s_abort = 1;
                        break;
                    }
                    uint8_t* st = smem + stage * kStageBytes;
#pragma unroll
                    for (int op = 0; op < 2; ++op) {
                        if (op == 0 ? !p.a_raw : !p.b_raw) continue;
                        float4* src = reinterpret_cast<float4*>(st + 2 * op * kTileBytes);
                        float4* dst = reinterpret_cast<float4*>(st + (2 * op + 1) * kTileBytes);
                        const bool mn = op == 0 ? p.a_mn : p.b_mn;
                        const int k_lim = kval - kb * kBK;  // MN-major: rows at or past it are zero
#pragma unroll 4
                        for (int i = ct; i < kTileBytes / 16; i += kConvThreads) {
                            float4 x = src[i];
                            if (mn && ((i >> 3) & 31) >= k_lim) {  // row (i / 8) % 32 of its 4 KB atom
                                x = make_float4(0.f, 0.f, 0.f, 0.f);
                                src[i] = x;
                            }
                            float4 lo;
                            lo.x = x.x - __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u);
                            lo.y = x.y - __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u);
                            lo.z = x.z - __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u);
                            lo.w = x.w - __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u);
                            dst[i] = lo;
                        }
                    }
                    fence_proxy_async_smem();  // the lo tiles are read by the tensor core
                    mbar_arrive(&conv[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
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
            const int64_t m = (int64_t)mt * kBM + q * 32 + lane;
            const int64_t gm = group_m(p, g);
            const bool row_ok = m < gm;
            // this warp's 32 rows for the staged stores
            const int64_t wrow0 = (int64_t)mt * kBM + q * 32;
            const int wrows = (int)(gm - wrow0 < 0 ? 0 : (gm - wrow0 > 32 ? 32 : gm - wrow0));
            float* cw = p.C + g * p.c_group_stride + wrow0 * p.ldc;
            float* crow = p.C + g * p.c_group_stride + m * p.ldc;
            const float* bias = p.bias ? p.bias + g * p.bias_group_stride : nullptr;
            const uint32_t t_row = tmem_base + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            auto process = [&](const int c, const uint32_t (&r)[32]) {
                const int64_t n0 = (int64_t)nt * p.n_mma + c * 32;
                if (p.tma_out) {
                    if (n0 >= p.N) return;  // the last tile's columns past N (warp-uniform)
                    // every row valid, whole 32-column chunks: the chunk goes to the warp's staging buffer
                    // in the map's 128-byte swizzled layout and one lane hands it to the TMA, which streams
                    // it out while the warp drains the next chunk
                    uint32_t* stg = s_stage[q];
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
#pragma unroll
                    for (int m4 = 0; m4 < 8; ++m4)
                        *reinterpret_cast<uint4*>(stg + lane * 32 + 4 * (m4 ^ (lane & 7))) =
                            make_uint4(r[4 * m4], r[4 * m4 + 1], r[4 * m4 + 2], r[4 * m4 + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmC, stg, (int32_t)n0, (int32_t)((int64_t)g * p.M + wrow0));
                        bulk_commit();
                    }
                    return;
                }
                if (p.epilogue != F32_EPI_SILU_MUL && p.vec_ok && n0 + 32 <= p.N) {
                    // row-contiguous stores through shared memory (see warp_store_chunk)
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float v = __uint_as_float(r[i]);
                        if ((p.epilogue == F32_EPI_BIAS || p.epilogue == F32_EPI_BIAS_GELU) && bias) v += bias[n0 + i];
                        if (p.epilogue == F32_EPI_BIAS_GELU) v = gelu_f(v);
                        w[i] = __float_as_uint(v);
                    }
                    warp_store_chunk<32>(s_stage[q], w, reinterpret_cast<uint8_t*>(cw + n0), p.ldc * 4, wrows, lane);
                    return;
                }
                if (!row_ok) return;
                if (p.vec_ok && n0 + 32 <= p.N) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float4 v = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                               __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                        float4* dst = reinterpret_cast<float4*>(crow + n0) + i;
                        if ((p.epilogue == F32_EPI_BIAS || p.epilogue == F32_EPI_BIAS_GELU) && bias) {
                            const float4 b = reinterpret_cast<const float4*>(bias + n0)[i];
                            v.x += b.x;
                            v.y += b.y;
                            v.z += b.z;
                            v.w += b.w;
                        }
                        if (p.epilogue == F32_EPI_BIAS_GELU) {
                            v.x = gelu_f(v.x);
                            v.y = gelu_f(v.y);
                            v.z = gelu_f(v.z);
                            v.w = gelu_f(v.w);
                        }
                        if (p.epilogue == F32_EPI_SILU_MUL) {
                            const float4 o = *dst;
                            v.x = silu_f(v.x) * o.x;
                            v.y = silu_f(v.y) * o.y;
                            v.z = silu_f(v.z) * o.z;
                            v.w = silu_f(v.w) * o.w;
                        }
                        *dst = v;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int64_t n = n0 + i;
                        if (n < p.N) {
                            float v = __uint_as_float(r[i]);
                            if ((p.epilogue == F32_EPI_BIAS || p.epilogue == F32_EPI_BIAS_GELU) && bias) v += bias[n];
                            if (p.epilogue == F32_EPI_BIAS_GELU) v = gelu_f(v);
                            if (p.epilogue == F32_EPI_SILU_MUL) v = silu_f(v) * crow[n];
                            crow[n] = v;
                        }
                    }
                }
            };
            // TMEM reads one chunk ahead of the math and stores
            const int nch = p.n_mma / 32;
            uint32_t ra[32], rb[32];
            tmem_ld32(t_row, ra);
            tmem_ld_wait(ra);
            for (int c = 0; c < nch; c += 2) {
                if (c + 1 < nch) tmem_ld32(t_row + (c + 1) * 32, rb);
                process(c, ra);
                if (c + 1 < nch) {
                    tmem_ld_wait(rb);
                    if (c + 2 < nch) tmem_ld32(t_row + (c + 2) * 32, ra);
                    process(c + 1, rb);
                    if (c + 2 < nch) tmem_ld_wait(ra);
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (s_abort) break;
        }
        if (p.tma_out && lane == 0) bulk_wait_all();  // the stores are done before the CTA exits
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kAccCols)
                     : "memory");
    }
}

struct SplitLayout {
    int64_t Kp;
    size_t a_bytes, b_bytes, total;  // each of hi/lo
};

SplitLayout split_layout(const F32Gemm& g) {
    SplitLayout l{};
    l.Kp = (g.K + kBK - 1) / kBK * kBK;
    l.a_bytes = align_up((size_t)g.groups * g.M * l.Kp * 4, 1024);
    l.b_bytes = align_up((size_t)g.groups * g.N * l.Kp * 4, 1024);
    l.total = 2 * (l.a_bytes + l.b_bytes);
    return l;
}

int launch_split(bool trans, bool bf16, const void* src, int64_t ld, int64_t gs, int groups, int64_t R, int64_t K,
                 int64_t Kp, const int32_t* krows, float* hi, float* lo, cudaStream_t stream) {
    MOE_REQUIRE(groups <= 65535 && (R + 31) / 32 <= 65535, MOE_ERR_UNSUPPORTED);
    const dim3 grid((unsigned)(Kp / 32), (unsigned)((R + 31) / 32), (unsigned)groups), block(32, 8);
    if (bf16) {
        const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src);
        if (trans) split_kernel<true><<<grid, block, 0, stream>>>(s, ld, gs, R, K, Kp, krows, hi, lo);
        else split_kernel<false><<<grid, block, 0, stream>>>(s, ld, gs, R, K, Kp, krows, hi, lo);
    } else {
        const float* s = static_cast<const float*>(src);
        if (trans) split_kernel<true><<<grid, block, 0, stream>>>(s, ld, gs, R, K, Kp, krows, hi, lo);
        else split_kernel<false><<<grid, block, 0, stream>>>(s, ld, gs, R, K, Kp, krows, hi, lo);
    }
    return launch_status();
}

}  // namespace

size_t tf32x3_workspace_size(const F32Gemm& g) {
    if (g.M < 1 || g.N < 1 || g.K < 1 || g.groups < 1) return 0;
    return split_layout(g).total;
}

int tf32x3_gemm_run(const F32Gemm& g, void* workspace, size_t workspace_bytes, int32_t* status,
                    cudaStream_t stream) {
    MOE_REQUIRE(g.A && g.B && g.C && g.M >= 1 && g.N >= 1 && g.K >= 1 && g.groups >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(g.groups <= kMaxGroups, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(g.rows_mode == 0 || g.rows != nullptr, MOE_ERR_INVALID_ARG);
    const SplitLayout l = split_layout(g);
    MOE_REQUIRE(workspace && aligned16(workspace) && workspace_bytes >= l.total, MOE_ERR_WORKSPACE);
    MOE_REQUIRE((int64_t)g.groups * g.M < (int64_t(1) << 31) && (int64_t)g.groups * g.N < (int64_t(1) << 31),
                MOE_ERR_UNSUPPORTED);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* a_hi = reinterpret_cast<float*>(ws);
    float* a_lo = reinterpret_cast<float*>(ws + l.a_bytes);
    float* b_hi = reinterpret_cast<float*>(ws + 2 * l.a_bytes);
    float* b_lo = reinterpret_cast<float*>(ws + 2 * l.a_bytes + l.b_bytes);
    const int32_t* krows = g.rows_mode == 2 ? g.rows : nullptr;

    // Raw operands (no split pass): fp32 with 16-byte aligned rows, and either K-major with contiguous
    // groups and no per-group K limit, or MN-major with a whole number of rows per group (rows past a
    // group's K limit are zeroed in the stage by the converter warps).
    const bool a_rawk = !g.a_bf16 && !g.a_trans && krows == nullptr && aligned16(g.A) && g.lda % 4 == 0 &&
                        g.lda >= g.K && (g.groups == 1 || g.a_group_stride == g.M * g.lda);
    const bool b_rawk = !g.b_bf16 && g.b_trans && krows == nullptr && aligned16(g.B) && g.ldb % 4 == 0 &&
                        g.ldb >= g.K && (g.groups == 1 || g.b_group_stride == g.N * g.ldb);
    const int64_t a_rpg = g.groups == 1 ? g.K : (g.lda > 0 ? g.a_group_stride / g.lda : 0);
    const int64_t b_rpg = g.groups == 1 ? g.K : (g.ldb > 0 ? g.b_group_stride / g.ldb : 0);
    const bool a_mn = kRawMnMajor && !g.a_bf16 && g.a_trans && aligned16(g.A) && g.lda % 4 == 0 && g.lda >= g.M &&
                      (g.groups == 1 || g.a_group_stride % g.lda == 0) && a_rpg >= g.K;
    const bool b_mn = kRawMnMajor && !g.b_bf16 && !g.b_trans && aligned16(g.B) && g.ldb % 4 == 0 && g.ldb >= g.N &&
                      (g.groups == 1 || g.b_group_stride % g.ldb == 0) && b_rpg >= g.K;
    const bool a_raw = a_rawk || a_mn, b_raw = b_rawk || b_mn;
    // The other operands are split beforehand, K-major: A as (groups, M, Kp), B^T as (groups, N, Kp)
    int rc = MOE_OK;
    if (!a_raw) {
        rc = launch_split(g.a_trans, g.a_bf16, g.A, g.lda, g.a_group_stride, g.groups, g.M, g.K, l.Kp, krows, a_hi,
                          a_lo, stream);
        if (rc != MOE_OK) return rc;
    }
    if (!b_raw) {
        rc = launch_split(!g.b_trans, g.b_bf16, g.B, g.ldb, g.b_group_stride, g.groups, g.N, g.K, l.Kp, krows, b_hi,
                          b_lo, stream);
        if (rc != MOE_OK) return rc;
    }

    T3Params kp{};
    kp.G = g.groups;
    kp.M = g.M;
    kp.N = g.N;
    const int64_t n32 = (g.N + 31) / 32 * 32;
    kp.n_mma = (int)(n32 < kBN ? n32 : kBN);
    kp.n_tiles = (int)((g.N + kp.n_mma - 1) / kp.n_mma);
    kp.k_blocks = (int)(l.Kp / kBK);
    kp.tx_bytes = (uint32_t)((a_raw ? 1 : 2) * kTileBytes + (b_raw ? 1 : 2) * kp.n_mma * kBK * 4);
    kp.a_raw = a_raw;
    kp.b_raw = b_raw;
    kp.a_mn = a_mn;
    kp.b_mn = b_mn;
    kp.a_rows_per_group = a_rpg;
    kp.b_rows_per_group = b_rpg;
    kp.krows = (a_mn || b_mn) ? krows : nullptr;
    kp.K = g.K;
    kp.rows = g.rows;
    kp.rows_mode = g.rows_mode;
    kp.C = g.C;
    kp.ldc = g.ldc;
    kp.c_group_stride = g.c_group_stride;
    kp.bias = g.bias;
    kp.bias_group_stride = g.bias_group_stride;
    kp.epilogue = g.epilogue;
    kp.vec_ok = aligned16(g.C) && g.ldc % 4 == 0 && g.c_group_stride % 4 == 0 &&
                (!g.bias || (aligned16(g.bias) && g.bias_group_stride % 4 == 0));
    // the weight-gradient form: plain fp32 out, all rows of every tile valid, groups back to back
    kp.tma_out = g.epilogue == F32_EPI_NONE && g.rows_mode != 1 && g.M % kBM == 0 && g.N % 32 == 0 && kp.vec_ok &&
                 g.c_group_stride == g.M * g.ldc && (int64_t)g.groups * g.M < (int64_t(1) << 31);
    kp.status = status;

    CUtensorMap mah, mal, mbh, mbl;
    if (a_mn) {  // the (K rows, M columns) operand in 32 x 32 boxes
        MOE_REQUIRE(make_map_f32_mn(&mah, g.A, g.M, (int64_t)g.groups * a_rpg, g.lda, 32), MOE_ERR_CUDA);
        mal = mah;
    } else if (a_raw) {  // the operand itself: K columns (zero fill up to Kp), row stride lda
        MOE_REQUIRE(make_map_f32(&mah, g.A, g.K, (int64_t)g.groups * g.M, g.lda, kBM), MOE_ERR_CUDA);
        mal = mah;
    } else {
        MOE_REQUIRE(make_map_f32(&mah, a_hi, l.Kp, (int64_t)g.groups * g.M, l.Kp, kBM), MOE_ERR_CUDA);
        MOE_REQUIRE(make_map_f32(&mal, a_lo, l.Kp, (int64_t)g.groups * g.M, l.Kp, kBM), MOE_ERR_CUDA);
    }
    if (b_mn) {
        MOE_REQUIRE(make_map_f32_mn(&mbh, g.B, g.N, (int64_t)g.groups * b_rpg, g.ldb, 32), MOE_ERR_CUDA);
        mbl = mbh;
    } else if (b_raw) {
        MOE_REQUIRE(make_map_f32(&mbh, g.B, g.K, (int64_t)g.groups * g.N, g.ldb, kp.n_mma), MOE_ERR_CUDA);
        mbl = mbh;
    } else {
        MOE_REQUIRE(make_map_f32(&mbh, b_hi, l.Kp, (int64_t)g.groups * g.N, l.Kp, kp.n_mma), MOE_ERR_CUDA);
        MOE_REQUIRE(make_map_f32(&mbl, b_lo, l.Kp, (int64_t)g.groups * g.N, l.Kp, kp.n_mma), MOE_ERR_CUDA);
    }

    CUtensorMap mc;
    if (kp.tma_out) MOE_REQUIRE(make_map_f32(&mc, g.C, g.N, (int64_t)g.groups * g.M, g.ldc, 32), MOE_ERR_CUDA);
    else mc = mah;  // unused

    const int64_t max_tiles = (int64_t)g.groups * ((g.M + kBM - 1) / kBM) * kp.n_tiles;
    MOE_REQUIRE(max_tiles < (int64_t(1) << 30), MOE_ERR_UNSUPPORTED);
    int grid = device_sm_count();
    if (max_tiles < grid) grid = (int)max_tiles;
    if (grid < 1) grid = 1;

    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 64 || !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes));
        if (dev < 64) attr_set[dev] = true;
    }
    tf32x3_kernel<<<grid, kThreads + kConvThreads, kSmemBytes, stream>>>(mah, mal, mbh, mbl, mc, kp);
    return launch_status();
}

}  // namespace moe
