// Router scores, softmax, stable top-k and gates in one kernel (bf16
// activations and router weight, fp32 accumulation in tensor memory).
//
// The router page's problem is one pass over the activations: s = x . W_r for
// every token, then a softmax and a top-k per token.  Writing s to memory and
// reading it back costs more than a quarter of the pass, so here the scores
// never leave the SM: each 128-token tile is multiplied on tcgen05 into a
// 128 x E fp32 accumulator in TMEM, and sixteen epilogue warps take it apart
// in registers.
//
// Work split: every CTA (one per SM) owns one contiguous run of tokens whose
// length is balanced to 32 rows across the grid, so no SM idles in a last
// partial wave; a run is processed in tiles of up to 128 tokens, and only the
// 32-row TMA boxes that hold the run's own rows are loaded.
//
// Warp roles (608 threads):
//   warp 0      TMA producer of the token rows: a 6-stage ring of 16 KB stages
//               (the deep ring keeps ~96 KB of activations in flight per SM,
//               what HBM latency needs at this SM's share of the bandwidth)
//   warp 1      TMA producer of the router weight: a 3-stage ring of E x 64
//               (the weight is re-read from L2 for every tile)
//   warp 2      TMEM owner and MMA issuer (one lane): two E-column
//               accumulators, so a tile's epilogue overlaps the next tile's
//               main loop
//   warps 3-18  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 tokens)
//               and one quarter of the E columns, 32 columns per TMEM load.
//               Pass 1 keeps the quarter's sorted top-8 (score desc, expert
//               index asc) and an online softmax sum; the four quarters' (max,
//               sum) pairs are combined through shared memory; pass 2 re-reads
//               the accumulator for the probabilities and then releases it.
//               The four top-8 lists are merged in two rounds, and the warp of
//               the first quarter writes selected, the gates and the counts.
// Per-expert probability sums are reduced over the 32 tokens of a warp with a
// fixed butterfly, kept in registers across tiles and added in a fixed order
// at the end, so prob_sum stays bitwise reproducible for a given grid.
//
// The exponentials use the fast intrinsic __expf.  Its documented error bound
// grows with |argument|; the arguments here are score differences (at most 0),
// so the error is largest on the smallest probabilities, whose absolute error
// stays far below the tolerances of the probability sums and the gates.
//
// Every mbarrier wait is bounded; after a timeout the producers and the MMA
// issuer stop, and the epilogue runs its remaining tiles without writing
// anything, so the named barriers between its warps always complete.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "route_fused.cuh"
#include "tc_gemm.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kRM = 128;       // tokens per tile (UMMA M)
constexpr int kRBK = 64;       // K per stage (64 bf16 = one 128-byte swizzle row)
constexpr int kRAStages = 6;
constexpr int kRBStages = 3;
constexpr int kRBox = 32;      // token rows per TMA box
constexpr int kREpiWarps = 16;
constexpr int kRThreads = (3 + kREpiWarps) * 32;
constexpr int kRABytes = kRM * kRBK * 2;  // 16 KB
constexpr int kRTopK = 8;

size_t fused_dyn_smem(int E) {
    return 1024 + (size_t)kRAStages * kRABytes + (size_t)kRBStages * E * kRBK * 2 + 256;
}

struct RFParams {
    int64_t T;
    int64_t units;  // ceil(T / 32)
    int k;
    int k_blocks;
    const float* bias;
    float* logits_out;
    int64_t* selected;
    void* gates;
    int gates_bf16;
    float* gates_f32;
    int32_t* part_counts;
    float* part_psum;
    int32_t* status;
};

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Insert (v, idx) into a list sorted by (score descending, index ascending).
// Every candidate has a higher index than the entries of equal score already in
// the list (a quarter's experts arrive in ascending order; a merged list's
// entries all lie above the receiving list's and arrive in its own order), so
// the new entry goes before the first strictly smaller score, and the entries
// from there on shift down by one place unconditionally: ties keep the lower
// expert index first.  The eight comparisons are independent of each other.
__device__ __forceinline__ void topk_insert(float (&tv)[kRTopK], int (&ti)[kRTopK], float v, int idx) {
    bool p[kRTopK];
#pragma unroll
    for (int j = 0; j < kRTopK; ++j) p[j] = v > tv[j];  // monotone: false ... false true ... true
#pragma unroll
    for (int j = kRTopK - 1; j >= 1; --j) {
        tv[j] = p[j] ? (p[j - 1] ? tv[j - 1] : v) : tv[j];
        ti[j] = p[j] ? (p[j - 1] ? ti[j - 1] : idx) : ti[j];
    }
    tv[0] = p[0] ? v : tv[0];
    ti[0] = p[0] ? idx : ti[0];
}

// Lane l returns the sum over the warp's lanes of a[l] (a is overwritten).
__device__ __forceinline__ float transpose_sum32(float* a, int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j) {
            const float send = up ? a[j] : a[j + o];
            const float keep = up ? a[j + o] : a[j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return a[0];
}

template <int CQ>
__global__ void __launch_bounds__(kRThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const RFParams p) {
    constexpr int E = 4 * CQ;
    constexpr int kBBytes = E * kRBK * 2;
    constexpr int NH = CQ / 32;  // 32-column chunks per quarter
    extern __shared__ uint8_t smem_raw[];
    __shared__ float s_red[2][4][kRM];          // per-quarter max and sum of each token
    __shared__ float s_cv[2][kRM][kRTopK];      // top-8 lists in transit: scores
    __shared__ int s_ci[2][kRM][kRTopK];        //                         indices
    __shared__ float s_bias[E];
    __shared__ int s_counts[E];
    __shared__ float s_psum[4][E];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smA = smem;
    uint8_t* smB = smA + kRAStages * kRABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + kRBStages * kBBytes);
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + kRAStages;
    uint64_t* b_full = bars + 2 * kRAStages;
    uint64_t* b_empty = bars + 2 * kRAStages + kRBStages;
    uint64_t* tfull = bars + 2 * kRAStages + 2 * kRBStages;
    uint64_t* tempty = tfull + 2;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // this CTA's run of tokens, balanced in 32-row units
    const int64_t u0 = (int64_t)blockIdx.x * p.units / gridDim.x;
    const int64_t u1 = (int64_t)(blockIdx.x + 1) * p.units / gridDim.x;
    const int64_t row_begin = u0 * kRBox;
    const int64_t row_end = u1 * kRBox < p.T ? u1 * kRBox : p.T;
    const int n_tiles = row_end > row_begin ? (int)((row_end - row_begin + kRM - 1) / kRM) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRAStages; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < kRBStages; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], kREpiWarps * 32);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(2 * E)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        s_bias[e] = p.bias ? p.bias[e] : 0.f;
        s_counts[e] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s_tmem;

    if (warp == 0) {
        // ------------------------- token-row producer -------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles && !s_abort; ++i) {
                const int64_t r0 = row_begin + (int64_t)i * kRM;
                const int64_t nrows = row_end - r0 < kRM ? row_end - r0 : kRM;
                const int nbox = (int)((nrows + kRBox - 1) / kRBox);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&a_empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&a_full[stage], (uint32_t)(nbox * kRBox * kRBK * 2));
                    uint8_t* dst = smA + stage * kRABytes;
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(dst + b * (kRBox * kRBK * 2), &tmX, kb * kRBK, (int32_t)(r0 + b * kRBox),
                                    &a_full[stage]);
                    if (++stage == kRAStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------ router-weight producer -----------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles && !s_abort; ++i) {
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&b_empty[stage], phase ^ 1u, p.status)) {
                        s_abort = 1;
                        break;
                    }
                    mbar_expect_tx(&b_full[stage], (uint32_t)kBBytes);
                    tma_load_2d(smB + stage * kBBytes, &tmW, kb * kRBK, 0, &b_full[stage]);
                    if (++stage == kRBStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------ MMA issuer -----------------------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(kRM, E);
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0;
            for (int i = 0; i < n_tiles && !s_abort; ++i) {
                const uint32_t acc = (uint32_t)i & 1u;
                if (!mbar_wait(&tempty[acc], (((uint32_t)i >> 1) & 1u) ^ 1u, p.status)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * E;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&a_full[sa], pa, p.status) || !mbar_wait(&b_full[sb], pb, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(smem_u32(smA + sa * kRABytes));
                    const uint64_t bd = sw128_desc(smem_u32(smB + sb * kBBytes));
#pragma unroll
                    for (int kk = 0; kk < kRBK / 16; ++kk)
                        tc_mma(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&a_empty[sa]);
                    tc_commit(&b_empty[sb]);
                    if (++sa == kRAStages) {
                        sa = 0;
                        pa ^= 1u;
                    }
                    if (++sb == kRBStages) {
                        sb = 0;
                        pb ^= 1u;
                    }
                }
                if (!ok) {
                    s_abort = 1;
                    break;
                }
                tc_commit(&tfull[acc]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue ------------------------------
        const int q = warp & 3;         // TMEM lane quarter this warp may read
        const int c = (warp - 3) >> 2;  // column quarter
        const int row = q * 32 + lane;
        const int bar_id = 1 + q;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float acc_ps[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) acc_ps[h] = 0.f;

        for (int i = 0; i < n_tiles; ++i) {
            const uint32_t acc = (uint32_t)i & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&tfull[acc], ((uint32_t)i >> 1) & 1u, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) s_abort = 1;
            tc_fence_after();
            const int64_t r0 = row_begin + (int64_t)i * kRM;
            const bool valid = r0 + row < row_end;
            const int64_t t = r0 + row;

            // pass 1, 32 columns at a time: bias, the quarter's top-8 (its experts in
            // ascending order) and an online softmax sum against the running max
            float tv[kRTopK];
            int ti[kRTopK];
#pragma unroll
            for (int j = 0; j < kRTopK; ++j) {
                tv[j] = -INFINITY;
                ti[j] = c * CQ + j;
            }
            float m_run = -INFINITY, ls = 0.f;
            bool finite = true;
            const bool write = valid && !s_abort;
            auto pass1 = [&](const int h) {
                uint32_t r[32];
                tmem_ld32(tmem_base + acc * E + lane_off + (uint32_t)(c * CQ + 32 * h), r);
                tmem_ld_wait(r);
                float v[32];
                const float4* b4 = reinterpret_cast<const float4*>(s_bias + c * CQ + 32 * h);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 b = b4[j4];
                    const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = 4 * j4 + u;
                        const float xv = __uint_as_float(r[j]) + bb[u];
                        const bool ok = fabsf(xv) < INFINITY;  // false for +-inf and NaN
                        finite = finite && ok;
                        v[j] = ok ? xv : -INFINITY;
                    }
                }
                if (p.logits_out && write) {
                    float4* dst = reinterpret_cast<float4*>(p.logits_out + t * E + c * CQ + 32 * h);
#pragma unroll
                    for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    topk_insert(tv, ti, v[j], c * CQ + 32 * h + j);
                    // branch-free: one exponential of -|xv - m_run| rescales the sum or adds the term
                    const float xv = v[j];
                    const float d = xv - m_run;
                    const float ed = xv == -INFINITY ? 0.f : __expf(-fabsf(d));
                    const bool up = d > 0.f;
                    ls = up ? fmaf(ls, ed, 1.0f) : ls + ed;
                    m_run = up ? xv : m_run;
                }
            };
            if constexpr (NH == 1) {
                pass1(0);
            } else {
#pragma unroll 1
                for (int h = 0; h < NH; ++h) pass1(h);
            }
            if (!finite && valid) set_status(p.status, MOE_ERR_NONFINITE);

            // softmax over all E: the quarters' (max, sum) pairs combined in a fixed order
            s_red[0][c][row] = m_run;
            s_red[1][c][row] = ls;
            named_bar(bar_id, 128);
            const float mx = fmaxf(fmaxf(s_red[0][0][row], s_red[0][1][row]), fmaxf(s_red[0][2][row], s_red[0][3][row]));
            float tot = 0.f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tot += s_red[1][cc][row] * __expf(s_red[0][cc][row] - mx);
            const float scale = valid ? __expf(m_run - mx) / tot : 0.f;

            // pass 2: probabilities, summed over the warp's 32 tokens per expert
            auto pass2 = [&](const int h) {
                uint32_t r[32];
                tmem_ld32(tmem_base + acc * E + lane_off + (uint32_t)(c * CQ + 32 * h), r);
                tmem_ld_wait(r);
                float pr[32];
                const float4* b4 = reinterpret_cast<const float4*>(s_bias + c * CQ + 32 * h);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 b = b4[j4];
                    const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = 4 * j4 + u;
                        const float xv = __uint_as_float(r[j]) + bb[u];
                        // scale is 0 for rows outside the run; a non-finite score contributes 0
                        pr[j] = fabsf(xv) < INFINITY ? __expf(xv - m_run) * scale : 0.f;
                    }
                }
                const float cs = transpose_sum32(pr, lane);
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) acc_ps[hh] += hh == h ? cs : 0.f;
            };
            if constexpr (NH == 1) {
                pass2(0);
            } else {
#pragma unroll 1
                for (int h = 0; h < NH; ++h) pass2(h);
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);  // the accumulator is no longer read: the next tile may use it

            // merge the four lists: (1 into 0, 3 into 2), then (2 into 0)
            if (c & 1) {
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) {
                    s_cv[c >> 1][row][j] = tv[j];
                    s_ci[c >> 1][row][j] = ti[j];
                }
            }
            named_bar(bar_id, 128);
            if (!(c & 1)) {
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) topk_insert(tv, ti, s_cv[c >> 1][row][j], s_ci[c >> 1][row][j]);
            }
            named_bar(bar_id, 128);
            if (c == 2) {
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) {
                    s_cv[0][row][j] = tv[j];
                    s_ci[0][row][j] = ti[j];
                }
            }
            named_bar(bar_id, 128);
            if (c == 0) {
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) topk_insert(tv, ti, s_cv[0][row][j], s_ci[0][row][j]);
                if (write) {
                    // gates: softmax of the selected scores (the first is the largest)
                    float ex[kRTopK];
                    float es = 0.f;
#pragma unroll
                    for (int j = 0; j < kRTopK; ++j) {
                        ex[j] = j < p.k ? __expf(tv[j] - tv[0]) : 0.f;
                        es += ex[j];
                    }
                    const float ginv = 1.0f / es;
#pragma unroll
                    for (int j = 0; j < kRTopK; ++j) {
                        if (j < p.k) {
                            const float g = ex[j] * ginv;
                            p.selected[t * p.k + j] = (int64_t)ti[j];
                            atomicAdd(&s_counts[ti[j]], 1);
                            if (p.gates_f32) p.gates_f32[t * p.k + j] = g;
                            if (p.gates) {
                                if (p.gates_bf16)
                                    reinterpret_cast<__nv_bfloat16*>(p.gates)[t * p.k + j] = __float2bfloat16_rn(g);
                                else
                                    reinterpret_cast<float*>(p.gates)[t * p.k + j] = g;
                            }
                        }
                    }
                }
            }
        }
        // per-CTA partials: the four lane quarters of each expert in a fixed order
#pragma unroll
        for (int h = 0; h < NH; ++h) s_psum[q][c * CQ + 32 * h + lane] = acc_ps[h];
        named_bar(5, kREpiWarps * 32);
        for (int e = threadIdx.x - 96; e < E; e += kREpiWarps * 32) {
            p.part_psum[(int64_t)blockIdx.x * E + e] = ((s_psum[0][e] + s_psum[1][e]) + s_psum[2][e]) + s_psum[3][e];
            p.part_counts[(int64_t)blockIdx.x * E + e] = s_counts[e];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * E) : "memory");
    }
}

template <int CQ>
int launch_fused(const CUtensorMap& mx, const CUtensorMap& mw, const RFParams& rp, int grid, cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    const size_t smem = fused_dyn_smem(4 * CQ);
    if (dev < 64 && !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(route_fused_kernel<CQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem));
        attr_set[dev] = true;
    }
    route_fused_kernel<CQ><<<grid, kRThreads, smem, stream>>>(mx, mw, rp);
    return launch_status();
}

}  // namespace

bool route_fused_supported(int64_t T, int64_t D, int64_t ldx, const void* x, const void* w_ed, int32_t E,
                           int32_t k) {
    return E == 256 && k >= 1 && k <= kRTopK && D >= 1 && D % 8 == 0 && ldx % 8 == 0 &&
           aligned16(x) && aligned16(w_ed) && T >= 1 && T < (int64_t(1) << 31);
}

int route_fused_grid(int64_t T) {
    const int64_t units = (T + kRBox - 1) / kRBox;
    const int sms = device_sm_count();
    return (int)(units < sms ? units : sms);
}

int route_fused_run(const void* x, int64_t T, int64_t D, int64_t ldx, const void* w_ed, int32_t E,
                    const float* bias, int32_t k, float* logits_out, int64_t* selected, void* gates, int gates_bf16,
                    float* gates_f32, int32_t* part_counts, float* part_psum, int32_t* status, cudaStream_t stream) {
    MOE_REQUIRE(route_fused_supported(T, D, ldx, x, w_ed, E, k), MOE_ERR_UNSUPPORTED);
    CUtensorMap mx, mw;
    MOE_REQUIRE(make_map(&mx, x, D, T, ldx, kRBox), MOE_ERR_CUDA);
    MOE_REQUIRE(make_map(&mw, w_ed, D, E, D, E), MOE_ERR_CUDA);
    RFParams rp{};
    rp.T = T;
    rp.units = (T + kRBox - 1) / kRBox;
    rp.k = k;
    rp.k_blocks = (int)((D + kRBK - 1) / kRBK);
    rp.bias = bias;
    rp.logits_out = logits_out;
    rp.selected = selected;
    rp.gates = gates;
    rp.gates_bf16 = gates_bf16;
    rp.gates_f32 = gates_f32;
    rp.part_counts = part_counts;
    rp.part_psum = part_psum;
    rp.status = status;
    const int grid = route_fused_grid(T);
    return launch_fused<64>(mx, mw, rp, grid, stream);
}

}  // namespace moe
