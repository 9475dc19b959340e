// moe_route and moe_aux_stats.
//
// Router scores come from the tensor-core GEMM (bf16, or split-tf32 for fp32),
// written as fp32 logits; then one warp per token does softmax, top-k and the
// renormalised gates entirely in registers, and each block leaves per-expert
// partial counts and probability sums that a second kernel adds up in a fixed
// order (so prob_sum is bitwise reproducible).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "route_fused.cuh"
#include "route_scores.cuh"
#include "f32_gemm.cuh"
#include "tc_gemm.cuh"
#include "tc_tf32.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;
constexpr int kRouteThreads = kRouteWarps * 32;
constexpr int kMaxRouteBlocks = 1024;  // bound on the per-block partials (workspace sizing)
// Blocks launched per SM (each warp then walks several tokens): the top-k kernel
// uses 80 registers, so three 256-thread blocks are resident per SM; a fourth
// only added a second partial wave (moe_route 197.6-198.6 against 201.0 us on
// the 65536-token router workload).
constexpr int kRouteBlocksPerSm = 3;
constexpr int kMaxK = 64;
constexpr int kMaxE = 1024;

int route_blocks(int64_t T) {
    int64_t b = (T + kRouteWarps - 1) / kRouteWarps;
    if (b < 2) b = 2;  // the fused kernel runs in CTA pairs
    return (int)(b < kMaxRouteBlocks ? b : kMaxRouteBlocks);
}

// Blocks the top-k kernel launches (<= route_blocks(T), the partials' capacity).
int topk_grid(int64_t T) {
    const int cap = kRouteBlocksPerSm * device_sm_count();
    const int b = route_blocks(T);
    return b < cap ? b : cap;
}

// SC: 0 softmax, 1 sigmoid clean scores.  SB: a selection bias is given
// (sel_bias (E), added to the clean scores for the selection only).  part_z
// (gridDim) or NULL: per-block sums of logsumexp(s_t)^2 for the router z-loss.
template <int EPL, typename InT, int SC, bool SB>
__global__ void __launch_bounds__(kRouteThreads)
    route_topk_kernel(const InT* __restrict__ logits, int64_t ld, int64_t T, int E, int k,
                      const float* __restrict__ bias, float* __restrict__ logits_out,
                      int64_t* __restrict__ selected, void* __restrict__ gates_out, int gates_bf16,
                      float* __restrict__ gates_f32, int32_t* __restrict__ part_counts,
                      float* __restrict__ part_psum, const float* __restrict__ sel_bias,
                      float* __restrict__ part_z, int32_t* status) {
    extern __shared__ float s_dyn[];
    float* s_psum = s_dyn;                                            // [kRouteWarps][E]
    int* s_counts = reinterpret_cast<int*>(s_psum + kRouteWarps * E);  // [E]
    __shared__ float s_z[kRouteWarps];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_counts[e] = 0;
    __syncthreads();

    float bias_r[EPL];
    float sbias_r[EPL];
    float psum[EPL];
#pragma unroll
    for (int m = 0; m < EPL; ++m) {
        const int e = m * 32 + lane;
        bias_r[m] = (bias && e < E) ? bias[e] : 0.f;
        sbias_r[m] = (SB && e < E) ? sel_bias[e] : 0.f;
        psum[m] = 0.f;
    }
    float zacc = 0.f;

    const int64_t stride = (int64_t)gridDim.x * kRouteWarps;
    // the next token's scores are loaded while the current token is processed
    InT nxt[EPL];
    int64_t t = (int64_t)blockIdx.x * kRouteWarps + warp;
    if (t < T) {
#pragma unroll
        for (int m = 0; m < EPL; ++m) nxt[m] = (m * 32 + lane < E) ? logits[t * ld + m * 32 + lane] : InT(0.f);
    }
    for (; t < T; t += stride) {
        InT cur[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) cur[m] = nxt[m];
        if (t + stride < T) {
            const InT* nrow = logits + (t + stride) * ld;
#pragma unroll
            for (int m = 0; m < EPL; ++m) nxt[m] = (m * 32 + lane < E) ? nrow[m * 32 + lane] : InT(0.f);
        }
        float v[EPL];
        uint32_t taken = 0;
        bool finite = true;
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            const int e = m * 32 + lane;
            if (e < E) {
                float x = to_f32(cur[m]) + bias_r[m];
                if (!isfinite(x)) {
                    finite = false;
                    x = -INFINITY;
                }
                v[m] = x;
                if (logits_out) logits_out[t * E + e] = x;
            } else {
                v[m] = -INFINITY;
                taken |= 1u << m;
            }
        }
        if (!__all_sync(0xffffffffu, finite) && lane == 0) set_status(status, MOE_ERR_NONFINITE);

        // clean scores: softmax over all experts (max-subtracted) or element-wise sigmoid
        float lmax = v[0];
#pragma unroll
        for (int m = 1; m < EPL; ++m) lmax = fmaxf(lmax, v[m]);
        const float smax = warp_max(lmax);
        float part = 0.f;
        float ex[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            const int e = m * 32 + lane;
            ex[m] = e < E ? expf(v[m] - smax) : 0.f;
            part += ex[m];
        }
        const float sum_exp = warp_sum(part);
        const float inv = 1.0f / sum_exp;
        float clean[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            const int e = m * 32 + lane;
            if (SC == 0) clean[m] = e < E ? ex[m] * inv : 0.f;
            else clean[m] = e < E ? sigmoid_stable_f(v[m]) : 0.f;
            psum[m] += clean[m];
        }
        if (part_z) {
            const float lse = smax + logf(sum_exp);
            zacc += lse * lse;
        }

        // top-k: k rounds of (lane-local best key, warp max of keys, lowest
        // index holding that key).  Keys preserve the float order exactly, so
        // equal scores tie and the index decides.  The key is the logit, or the
        // clean score plus the selection bias when one is given.
        uint32_t key[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            const int e = m * 32 + lane;
            key[m] = (e < E) ? order_key(SB ? clean[m] + sbias_r[m] : v[m]) : 0u;
        }
        // Winner j is kept by lane j (j < 32) or lane j - 32 in registers; the
        // rounds contain no divergent branch and no memory access.
        uint32_t sel0 = 0, sel1 = 0;
        float val0 = 0.f, val1 = 0.f;
        for (int j = 0; j < k; ++j) {
            uint32_t lk = 0;  // below every finite or infinite key
            uint32_t li = 0xffffffffu;
            float lv = 0.f;
#pragma unroll
            for (int m = 0; m < EPL; ++m) {
                const bool live = !((taken >> m) & 1u);
                if (live && key[m] > lk) {  // ascending m: the first of equal keys keeps the lowest index
                    lk = key[m];
                    li = (uint32_t)(m * 32 + lane);
                    lv = v[m];
                }
            }
            const uint32_t gk = __reduce_max_sync(0xffffffffu, lk);
            const uint32_t bi = __reduce_min_sync(0xffffffffu, lk == gk ? li : 0xffffffffu);
            const int wl = (int)(bi & 31u);
            // the winner's raw logit: its key when ranking by logit, else from the winning lane
            const float wv = SB ? __shfl_sync(0xffffffffu, lv, wl) : key_to_float(gk);
            taken |= wl == lane ? 1u << (bi >> 5) : 0u;
            if (j < 32) {
                sel0 = lane == j ? bi : sel0;
                val0 = lane == j ? wv : val0;
            } else {
                sel1 = lane == j - 32 ? bi : sel1;
                val1 = lane == j - 32 ? wv : val1;
            }
        }
        if (lane < k) {
            selected[t * k + lane] = (int64_t)sel0;
            atomicAdd(&s_counts[sel0], 1);
        }
        if (lane + 32 < k) {
            selected[t * k + lane + 32] = (int64_t)sel1;
            atomicAdd(&s_counts[sel1], 1);
        }

        // gates: softmax of the selected logits, or of their log-sigmoids (k <= 64:
        // each lane owns j = lane and j = lane + 32)
        float w0 = -INFINITY, w1 = -INFINITY;
        if (lane < k) w0 = SC == 0 ? val0 : log_sigmoid_f(val0);
        if (lane + 32 < k) w1 = SC == 0 ? val1 : log_sigmoid_f(val1);
        const float wmax = warp_max(fmaxf(w0, w1));
        const float e0 = lane < k ? expf(w0 - wmax) : 0.f;
        const float e1 = lane + 32 < k ? expf(w1 - wmax) : 0.f;
        const float ginv = 1.0f / warp_sum(e0 + e1);
        for (int j = lane; j < k; j += 32) {
            const float g = (j == lane ? e0 : e1) * ginv;
            if (gates_f32) gates_f32[t * k + j] = g;
            if (gates_out) {
                if (gates_bf16) reinterpret_cast<__nv_bfloat16*>(gates_out)[t * k + j] = __float2bfloat16_rn(g);
                else reinterpret_cast<float*>(gates_out)[t * k + j] = g;
            }
        }
        __syncwarp();
    }

    // block partials in a fixed order: warps 0..7, then per block slot
#pragma unroll
    for (int m = 0; m < EPL; ++m) {
        const int e = m * 32 + lane;
        if (e < E) s_psum[warp * E + e] = psum[m];
    }
    if (lane == 0) s_z[warp] = zacc;
    __syncthreads();
    if (part_z && threadIdx.x == 0) {
        float z = 0.f;
        for (int w = 0; w < kRouteWarps; ++w) z += s_z[w];
        part_z[blockIdx.x] = z;
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float s = 0.f;
        for (int w = 0; w < kRouteWarps; ++w) s += s_psum[w * E + e];
        part_psum[(int64_t)blockIdx.x * E + e] = s;
        part_counts[(int64_t)blockIdx.x * E + e] = s_counts[e];
    }
}

// counts[e] and prob_sum[e] = fixed-order sums of the block partials.  A block
// owns 32 consecutive experts (coalesced loads across experts); its 32 warps
// each add every 32nd partial row in ascending order, then warp 0 adds the 32
// warp sums in order.  The order depends only on the partial count, so the
// result is bitwise reproducible.
constexpr int kReduceWarps = 32;

__global__ void __launch_bounds__(kReduceWarps * 32)
    route_reduce_kernel(const int32_t* __restrict__ part_counts, const float* __restrict__ part_psum, int nblocks,
                        int E, int32_t* __restrict__ counts, float* __restrict__ prob_sum,
                        const float* __restrict__ part_z, int64_t T, float* __restrict__ z_loss) {
    __shared__ float s_p[kReduceWarps][32];
    __shared__ int s_c[kReduceWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 32 + lane;
    int c = 0;
    float s = 0.f;
    if (e < E) {
#pragma unroll 8
        for (int b = warp; b < nblocks; b += kReduceWarps) {
            c += part_counts[(int64_t)b * E + e];
            s += part_psum[(int64_t)b * E + e];
        }
    }
    s_p[warp][lane] = s;
    s_c[warp][lane] = c;
    __syncthreads();
    if (warp == 0 && e < E) {
        float ts = 0.f;
        int tc = 0;
        for (int w = 0; w < kReduceWarps; ++w) {
            ts += s_p[w][lane];
            tc += s_c[w][lane];
        }
        counts[e] = tc;
        prob_sum[e] = ts;
    }
    // router z-loss: the block partials in ascending order, divided by T
    if (part_z && blockIdx.x == 0 && threadIdx.x == 0) {
        float z = 0.f;
        for (int b = 0; b < nblocks; ++b) z += part_z[b];
        *z_loss = z / (float)T;
    }
}

template <typename InT>
int launch_topk(int epl, const InT* logits, int64_t ld, int64_t T, int E, int k, const float* bias,
                float* logits_out, int64_t* selected, void* gates, int gates_bf16, float* gates_f32,
                int32_t* part_counts, float* part_psum, int scoring, const float* sel_bias, float* part_z,
                int32_t* status, cudaStream_t stream) {
    const int nb = topk_grid(T);
    const size_t smem = sizeof(float) * (size_t)kRouteWarps * E + sizeof(int) * (size_t)E;
#define MOE_TOPK_CASE(N)                                                                                      \
    case N: {                                                                                                 \
        auto kern = scoring == 0 ? (sel_bias ? route_topk_kernel<N, InT, 0, true> : route_topk_kernel<N, InT, 0, false>) \
                                 : (sel_bias ? route_topk_kernel<N, InT, 1, true> : route_topk_kernel<N, InT, 1, false>); \
        if (smem > 48 * 1024)                                                                                 \
            MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); \
        kern<<<nb, kRouteThreads, smem, stream>>>(logits, ld, T, E, k, bias, logits_out, selected, gates,     \
                                                  gates_bf16, gates_f32, part_counts, part_psum, sel_bias,    \
                                                  part_z, status);                                            \
        break;                                                                                                \
    }
    switch (epl) {
        MOE_TOPK_CASE(1)
        MOE_TOPK_CASE(2)
        MOE_TOPK_CASE(4)
        MOE_TOPK_CASE(8)
        MOE_TOPK_CASE(16)
        MOE_TOPK_CASE(32)
        default: return MOE_ERR_UNSUPPORTED;
    }
#undef MOE_TOPK_CASE
    return launch_status();
}

int epl_for(int E) {
    int epl = 1;
    while (epl * 32 < E) epl *= 2;
    return epl;
}

struct RouteWs {
    size_t logits_off, wt_off, pc_off, pp_off, pz_off, split_off, total;
};

// The fp32 router GEMM in F32Gemm form (operands filled in by the caller).
F32Gemm router_f32_shape(int64_t T, int64_t D, int32_t E) {
    F32Gemm g{};
    g.M = T;
    g.N = E;
    g.K = D;
    g.groups = 1;
    return g;
}

RouteWs route_ws_layout(int64_t T, int64_t D, int32_t E, moe_dtype dtype, int has_w, moe_router_layout layout) {
    RouteWs w{};
    size_t off = 0;
    w.logits_off = off;
    if (has_w) off += align_up((size_t)T * E * sizeof(float), 256);
    w.wt_off = off;
    if (has_w && dtype == MOE_BF16 && layout == MOE_ROUTER_DE) off += align_up((size_t)E * D * 2, 256);
    const int nb = route_blocks(T);
    w.pc_off = off;
    off += align_up((size_t)nb * E * sizeof(int32_t), 256);
    w.pp_off = off;
    off += align_up((size_t)nb * E * sizeof(float), 256);
    w.pz_off = off;
    off += align_up((size_t)nb * sizeof(float), 256);
    w.split_off = off;
    if (has_w && dtype == MOE_F32) off += align_up(tf32x3_workspace_size(router_f32_shape(T, D, E)), 256);
    w.total = off;
    return w;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_route_workspace_size(int64_t T, int64_t D, int32_t E, moe_dtype dtype, int has_router_weight,
                                           moe_router_layout layout) {
    if (T < 1 || E < 1) return 0;
    return route_ws_layout(T, D, E, dtype, has_router_weight, layout).total;
}

extern "C" int moe_route_ex(const void* x, moe_dtype dtype, int64_t T, int64_t D, int64_t ldx,
                            const void* w_router, moe_router_layout layout, int32_t E, const float* logit_bias,
                            int32_t k, moe_scoring scoring, const float* selection_bias, float* logits_out,
                            int64_t* selected, void* gates, float* gates_f32, int32_t* counts, float* prob_sum,
                            float* z_loss, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                            moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(valid_dtype(dtype), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(x && selected && counts && prob_sum, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && E >= 1 && k >= 1 && k <= E, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(E <= kMaxE && k <= kMaxK, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(layout == MOE_ROUTER_DE || layout == MOE_ROUTER_ED, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(scoring == MOE_SCORE_SOFTMAX || scoring == MOE_SCORE_SIGMOID, MOE_ERR_INVALID_ARG);
    const int has_w = w_router != nullptr;
    if (has_w) MOE_REQUIRE(D >= 1 && ldx >= D, MOE_ERR_INVALID_ARG);
    else MOE_REQUIRE(ldx >= E, MOE_ERR_INVALID_ARG);
    const RouteWs wl = route_ws_layout(T, D, E, dtype, has_w, layout);
    MOE_REQUIRE(workspace != nullptr && workspace_bytes >= wl.total, MOE_ERR_WORKSPACE);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* part_counts = reinterpret_cast<int32_t*>(ws + wl.pc_off);
    float* part_psum = reinterpret_cast<float*>(ws + wl.pp_off);
    float* part_z = z_loss ? reinterpret_cast<float*>(ws + wl.pz_off) : nullptr;
    const int sc = scoring == MOE_SCORE_SIGMOID ? 1 : 0;
    const int epl = epl_for(E);
    const int gates_bf16 = dtype == MOE_BF16;
    int rc = MOE_OK;
    int nb = topk_grid(T);

    // bf16 softmax router without the variants: scores, softmax, top-k and gates in one kernel
    if (has_w && dtype == MOE_BF16 && sc == 0 && selection_bias == nullptr && z_loss == nullptr &&
        (logits_out == nullptr || aligned16(logits_out))) {
        const void* w_ed = w_router;
        if (layout == MOE_ROUTER_DE) w_ed = ws + wl.wt_off;
        if (route_fused_supported(T, D, ldx, x, w_ed, E, k)) {
            if (layout == MOE_ROUTER_DE) {
                rc = transpose_matrices(w_router, ws + wl.wt_off, 1, D, E, MOE_BF16, stream);
                if (rc != MOE_OK) return rc;
            }
            rc = route_fused_run(x, T, D, ldx, w_ed, E, logit_bias, k, logits_out, selected, gates, gates_bf16,
                                 gates_f32, part_counts, part_psum, dev_status, stream);
            if (rc != MOE_OK) return rc;
            nb = route_fused_grid(T);
            route_reduce_kernel<<<(E + 31) / 32, kReduceWarps * 32, 0, stream>>>(part_counts, part_psum, nb, E,
                                                                                 counts, prob_sum, nullptr, T,
                                                                                 nullptr);
            return launch_status();
        }
    }

    if (has_w) {
        // scores s = x . W (+ bias) into fp32 logits
        float* lg = logits_out ? logits_out : reinterpret_cast<float*>(ws + wl.logits_off);
        if (dtype == MOE_BF16) {
            const void* w_ed = w_router;
            if (layout == MOE_ROUTER_DE) {
                void* wt = ws + wl.wt_off;
                rc = transpose_matrices(w_router, wt, 1, D, E, MOE_BF16, stream);
                if (rc != MOE_OK) return rc;
                w_ed = wt;
            }
            // tokens on the MMA's M side, all E experts in one N tile
            TcGemmProblem q{};
            q.a = x;
            q.lda = ldx;
            q.a_rows_total = T;
            q.a_rows_per_group = 0;
            q.b = w_ed;
            q.ldb = D;
            q.b_rows_total = E;
            q.b_rows_per_group = 0;
            q.G = 1;
            q.M = T;
            q.N = E;
            q.K = D;
            q.rows = nullptr;
            q.out = lg;
            q.ldo = E;
            q.out_rows_per_group = 0;
            q.bias = logit_bias;
            q.epilogue = TC_EPI_F32;
            q.status = dev_status;
            rc = tc_gemm_run(q, stream);
        } else {
            F32Gemm g{};
            g.A = static_cast<const float*>(x);
            g.lda = ldx;
            g.a_trans = false;
            g.B = static_cast<const float*>(w_router);
            // B(k=d, n=e): (D,E) row-major is "not transposed"; (E,D) is transposed.
            g.b_trans = layout == MOE_ROUTER_ED;
            g.ldb = layout == MOE_ROUTER_ED ? D : E;
            g.C = lg;
            g.ldc = E;
            g.M = T;
            g.N = E;
            g.K = D;
            g.groups = 1;
            g.bias = logit_bias;
            g.epilogue = F32_EPI_BIAS;
            rc = tf32x3_gemm_run(g, ws + wl.split_off, wl.total - wl.split_off, dev_status, stream);
        }
        if (rc != MOE_OK) return rc;
        rc = launch_topk<float>(epl, lg, E, T, E, k, nullptr, nullptr, selected, gates, gates_bf16, gates_f32,
                                part_counts, part_psum, sc, selection_bias, part_z, dev_status, stream);
    } else if (dtype == MOE_BF16) {
        rc = launch_topk<__nv_bfloat16>(epl, static_cast<const __nv_bfloat16*>(x), ldx, T, E, k, logit_bias,
                                        logits_out, selected, gates, gates_bf16, gates_f32, part_counts, part_psum,
                                        sc, selection_bias, part_z, dev_status, stream);
    } else {
        rc = launch_topk<float>(epl, static_cast<const float*>(x), ldx, T, E, k, logit_bias, logits_out, selected,
                                gates, gates_bf16, gates_f32, part_counts, part_psum, sc, selection_bias, part_z,
                                dev_status, stream);
    }
    if (rc != MOE_OK) return rc;
    route_reduce_kernel<<<(E + 31) / 32, kReduceWarps * 32, 0, stream>>>(part_counts, part_psum, nb, E, counts,
                                                                         prob_sum, part_z, T, z_loss);
    return launch_status();
}

extern "C" int moe_route(const void* x, moe_dtype dtype, int64_t T, int64_t D, int64_t ldx, const void* w_router,
                         moe_router_layout layout, int32_t E, const float* logit_bias, int32_t k, float* logits_out,
                         int64_t* selected, void* gates, float* gates_f32, int32_t* counts, float* prob_sum,
                         int32_t* dev_status, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    return moe_route_ex(x, dtype, T, D, ldx, w_router, layout, E, logit_bias, k, MOE_SCORE_SOFTMAX, nullptr,
                        logits_out, selected, gates, gates_f32, counts, prob_sum, nullptr, dev_status, workspace,
                        workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// moe_renormalize_kept_gates
// ---------------------------------------------------------------------------
namespace moe {
namespace {

__global__ void renormalize_kernel(const float* __restrict__ gates, const int64_t* __restrict__ slot, int64_t T,
                                   int k, float* __restrict__ out) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    float mass = 0.f;
    for (int j = 0; j < k; ++j)
        if (slot[t * k + j] >= 0) mass += gates[t * k + j];
    const float inv = mass > 0.f ? 1.0f / mass : 0.f;
    for (int j = 0; j < k; ++j) out[t * k + j] = slot[t * k + j] >= 0 ? gates[t * k + j] * inv : 0.f;
}

}  // namespace
}  // namespace moe

extern "C" int moe_renormalize_kept_gates(const float* gates_f32, const int64_t* slot, int64_t T, int32_t k,
                                          float* out, moe_stream_t stream) {
    MOE_REQUIRE(gates_f32 && slot && out && T >= 1 && k >= 1, MOE_ERR_INVALID_ARG);
    renormalize_kernel<<<(unsigned)((T + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        gates_f32, slot, T, k, out);
    return launch_status();
}

// ---------------------------------------------------------------------------
// moe_aux_stats
// ---------------------------------------------------------------------------
namespace moe {
namespace {

__global__ void aux_stats_kernel(const int32_t* __restrict__ counts, const float* __restrict__ prob_sum, int64_t T,
                                 int E, float kn, float aux_coef, void* f_out, void* P_out, int out_bf16,
                                 float* aux) {
    __shared__ float s_red[1024];
    float acc = 0.f;
    const float invT = 1.0f / (float)T;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const float c = (float)counts[e];
        const float f = c * invT;
        const float P = prob_sum[e] * invT;
        if (out_bf16) {
            reinterpret_cast<__nv_bfloat16*>(f_out)[e] = __float2bfloat16_rn(f);
            reinterpret_cast<__nv_bfloat16*>(P_out)[e] = __float2bfloat16_rn(P);
        } else {
            reinterpret_cast<float*>(f_out)[e] = f;
            reinterpret_cast<float*>(P_out)[e] = P;
        }
        acc += (c / ((float)T * kn)) * P;
    }
    s_red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) s_red[threadIdx.x] += s_red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const float a = (float)E * s_red[0];
        aux[0] = a;
        aux[1] = aux_coef * a;
    }
}

}  // namespace
}  // namespace moe

extern "C" int moe_aux_stats(const int32_t* counts, const float* prob_sum, int64_t T, int32_t E, int32_t k,
                             int normalize_by_k, float aux_coef, void* f, void* P, moe_dtype out_dtype, float* aux,
                             moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(counts && prob_sum && f && P && aux, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && E >= 1 && k >= 1 && valid_dtype(out_dtype), MOE_ERR_INVALID_ARG);
    aux_stats_kernel<<<1, 1024, 0, stream>>>(counts, prob_sum, T, E, normalize_by_k ? (float)k : 1.0f, aux_coef, f, P,
                                             out_dtype == MOE_BF16, aux);
    return launch_status();
}

// ---------------------------------------------------------------------------
// moe_router_backward
// ---------------------------------------------------------------------------
namespace moe {
namespace {

// Column sums of g (T, E) in a fixed order, in two passes.  Pass 1: block
// (b, c) covers experts 32b + lane over the rows of chunk c; warp w adds rows
// t = chunk start + w, + 32, ..., warp 0 adds the 32 warp sums into part[c][e].
// Pass 2: out[e] = sum over the chunks in ascending order (plus add[s][e] of
// `nadd` further partial rows when given).
constexpr int kColChunks = 64;
__global__ void __launch_bounds__(1024)
    column_sum_part_kernel(const float* __restrict__ g, int64_t T, int E, int64_t chunk, float* __restrict__ part) {
    __shared__ float s[32][33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 32 + lane;
    const int64_t t0 = (int64_t)blockIdx.y * chunk;
    const int64_t t1 = t0 + chunk < T ? t0 + chunk : T;
    float acc = 0.f;
    if (e < E)
        for (int64_t t = t0 + warp; t < t1; t += 32) acc += g[t * E + e];
    s[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && e < E) {
        float tot = 0.f;
        for (int w = 0; w < 32; ++w) tot += s[w][lane];
        part[(int64_t)blockIdx.y * E + e] = tot;
    }
}

// out[i] = sum_{s < n} part[s][i], s ascending (i < len).
__global__ void sum_rows_kernel(const float* __restrict__ part, int n, int64_t len, float* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < len; i += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int s = 0; s < n; ++s) acc += part[(int64_t)s * len + i];
        out[i] = acc;
    }
}

// K splits of the weight-gradient product (reduction over the T tokens): enough
// tiles for the SMs while T splits evenly.
int wgrad_splits(int64_t T, int64_t M, int64_t N) {
    const int64_t tiles = ((M + 127) / 128) * ((N + 127) / 128);
    int s = 1;
    while (s < 8 && tiles * s * 2 <= 160 && T % (2 * s) == 0 && T / (2 * s) >= 512) s *= 2;
    return s;
}

// The two GEMMs of the router backward in F32Gemm form.
void router_bwd_gemms(moe_dtype dtype, const void* x, int64_t T, int64_t D, int64_t ldx, const void* w,
                      moe_router_layout layout, int32_t E, const float* g, float* dx, float* dw, F32Gemm& gx,
                      F32Gemm& gw) {
    const bool bf16 = dtype == MOE_BF16;
    // dx[t,d] = sum_e g[t,e] W(e,d)
    gx = F32Gemm{};
    gx.A = g;
    gx.lda = E;
    gx.B = static_cast<const float*>(w);
    gx.b_bf16 = bf16;
    if (layout == MOE_ROUTER_ED) {  // W(e,d) = w[e*D + d]: B(k=e, n=d) not transposed
        gx.ldb = D;
        gx.b_trans = false;
    } else {  // W(e,d) = w[d*E + e]: B(k=e, n=d) = w[n*E + k]
        gx.ldb = E;
        gx.b_trans = true;
    }
    gx.C = dx;
    gx.ldc = D;
    gx.M = T;
    gx.N = D;
    gx.K = E;
    // dw in the weight's layout; reduction over t
    gw = F32Gemm{};
    if (layout == MOE_ROUTER_ED) {  // dw[e,d] = sum_t g[t,e] x[t,d]
        gw.A = g;
        gw.lda = E;
        gw.a_trans = true;
        gw.B = static_cast<const float*>(x);
        gw.b_bf16 = bf16;
        gw.ldb = ldx;
        gw.M = E;
        gw.N = D;
        gw.ldc = D;
    } else {  // dw[d,e] = sum_t x[t,d] g[t,e]
        gw.A = static_cast<const float*>(x);
        gw.a_bf16 = bf16;
        gw.lda = ldx;
        gw.a_trans = true;
        gw.B = g;
        gw.ldb = E;
        gw.M = D;
        gw.N = E;
        gw.ldc = E;
    }
    gw.C = dw;
    gw.K = T;
    // split the reduction over t into S groups of T/S rows, partial products summed afterwards
    const int S = wgrad_splits(T, gw.M, gw.N);
    if (S > 1) {
        gw.groups = S;
        gw.K = T / S;
        if (layout == MOE_ROUTER_ED) {
            gw.a_group_stride = gw.K * E;
            gw.b_group_stride = gw.K * ldx;
        } else {
            gw.a_group_stride = gw.K * ldx;
            gw.b_group_stride = gw.K * E;
        }
        gw.c_group_stride = gw.M * gw.N;
    }
}

// Workspace of the router backward: the split operands, then (when the
// weight gradient is split) the partial products, then the column-sum partials.
struct RouterBwdWs {
    size_t split, partials, colsum, total;
};

RouterBwdWs router_bwd_layout(const F32Gemm& gx, const F32Gemm& gw, int32_t E) {
    RouterBwdWs l{};
    const size_t a = tf32x3_workspace_size(gx), b = tf32x3_workspace_size(gw);
    l.split = align_up(a > b ? a : b, 256);
    l.partials = gw.groups > 1 ? align_up((size_t)gw.groups * gw.M * gw.N * 4, 256) : 0;
    l.colsum = align_up((size_t)kColChunks * E * 4, 256);
    l.total = l.split + l.partials + l.colsum;
    return l;
}

// ---- the bf16 router backward: dlogits in three bf16 parts on the bf16 tensor cores ----
//
// x and W_r in bf16 are exact in any wider format, so the only operand that
// needs more than bf16 is dlogits (fp32).  It is split as g = g1 + g2 + g3
// with g1 = bf16(g), g2 = bf16(g - g1), g3 = bf16(g - g1 - g2): 24 mantissa bits
// in all, each product g_i * x (or g_i * W) exact in the fp32 accumulator.  So
//   dx = [g1 | g2 | g3] . [W; W; W]     one bf16 GEMM with K = 3E
//   dW = sum_i g_i^T x                  three bf16 GEMMs reading g_i in place,
//                                       the reduction over the tokens split in S
//                                       groups, all partials summed in a fixed order.

__global__ void split3_bf16_kernel(const float* __restrict__ g, int64_t n, int E, __nv_bfloat16* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / E;
        const int e = (int)(i - t * E);
        const float v = g[i];
        const __nv_bfloat16 h1 = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(h1);
        const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(h2);
        __nv_bfloat16* row = out + t * 3 * E;
        row[e] = h1;
        row[E + e] = h2;
        row[2 * E + e] = __float2bfloat16_rn(r2);
    }
}

// token groups of the weight gradient (each a multiple of 64 tokens, so no group
// reads into the next); one group when T is not a multiple of 64
int router_bwd_bf16_groups(int64_t T) {
    int s = 1;
    while (s < 8 && T % (128 * s) == 0 && T / (2 * s) >= 1024) s *= 2;
    return s;
}

bool router_bwd_bf16_shape_ok(int64_t D, int32_t E) { return E % 64 == 0 && D % 64 == 0; }

struct RouterBwdBf16Ws {
    size_t parts, wrep, partials, colsum, total;
};

RouterBwdBf16Ws router_bwd_bf16_layout(int64_t T, int64_t D, int32_t E) {
    RouterBwdBf16Ws l{};
    size_t off = 0;
    l.parts = off;
    off += align_up((size_t)T * 3 * E * 2, 256);
    l.wrep = off;
    off += align_up((size_t)3 * E * D * 2, 256);
    l.partials = off;
    off += align_up((size_t)3 * router_bwd_bf16_groups(T) * E * D * 4, 256);
    l.colsum = off;
    off += align_up((size_t)kColChunks * E * 4, 256);
    l.total = off;
    return l;
}

int router_backward_bf16(const void* x, int64_t T, int64_t D, int64_t ldx, const void* w, moe_router_layout layout,
                         int32_t E, const float* dlogits, float* dx, float* dw, int32_t* status, uint8_t* ws,
                         const RouterBwdBf16Ws& l, cudaStream_t stream) {
    __nv_bfloat16* parts = reinterpret_cast<__nv_bfloat16*>(ws + l.parts);
    {
        const int64_t n = T * E;
        const int64_t nb = (n + 255) / 256;
        split3_bf16_kernel<<<(unsigned)(nb < 8192 ? nb : 8192), 256, 0, stream>>>(dlogits, n, E, parts);
        const int rc = launch_status();
        if (rc != MOE_OK) return rc;
    }
    const bool ed = layout == MOE_ROUTER_ED;
    if (dx) {
        // [W; W; W] along K in the weight's own orientation
        __nv_bfloat16* wrep = reinterpret_cast<__nv_bfloat16*>(ws + l.wrep);
        for (int i = 0; i < 3; ++i) {
            if (ed)
                MOE_CUDA_TRY(cudaMemcpyAsync(wrep + (int64_t)i * E * D, w, (size_t)E * D * 2, cudaMemcpyDeviceToDevice,
                                             stream));
            else
                MOE_CUDA_TRY(cudaMemcpy2DAsync(wrep + (int64_t)i * E, (size_t)3 * E * 2, w, (size_t)E * 2,
                                               (size_t)E * 2, (size_t)D, cudaMemcpyDeviceToDevice, stream));
        }
        TcGemmProblem q{};
        q.a = parts;
        q.lda = 3 * E;
        q.a_rows_total = T;
        q.b = wrep;
        if (ed) {  // B(k, n) = wrep[k * D + n]
            q.b_mn_major = true;
            q.ldb = D;
            q.b_rows_total = 3 * E;
            q.b_rows_per_group = 3 * E;
        } else {  // B(k, n) = wrep[n * 3E + k]
            q.ldb = 3 * E;
            q.b_rows_total = D;
        }
        q.G = 1;
        q.M = T;
        q.N = D;
        q.K = 3 * E;
        q.out = dx;
        q.ldo = D;
        q.out_rows_per_group = T;
        q.epilogue = TC_EPI_F32;
        q.status = status;
        const int rc = tc_gemm_run(q, stream);
        if (rc != MOE_OK) return rc;
    }
    if (dw) {
        const int S = router_bwd_bf16_groups(T);
        const int64_t tg = T / S;
        float* part = reinterpret_cast<float*>(ws + l.partials);
        for (int i = 0; i < 3; ++i) {
            TcGemmProblem q{};
            q.a_mn_major = true;
            q.b_mn_major = true;
            q.G = S;
            q.K = tg;
            if (ed) {  // dw[e, d] = sum_t g_i[t, e] x[t, d]
                q.a = parts + (int64_t)i * E;
                q.lda = 3 * E;
                q.M = E;
                q.b = x;
                q.ldb = ldx;
                q.N = D;
            } else {  // dw[d, e] = sum_t x[t, d] g_i[t, e]
                q.a = x;
                q.lda = ldx;
                q.M = D;
                q.b = parts + (int64_t)i * E;
                q.ldb = 3 * E;
                q.N = E;
            }
            q.a_rows_total = T;
            q.a_rows_per_group = tg;
            q.b_rows_total = T;
            q.b_rows_per_group = tg;
            q.out = part + (int64_t)i * S * E * D;
            q.ldo = q.N;
            q.out_rows_per_group = q.M;
            q.epilogue = TC_EPI_F32;
            q.status = status;
            const int rc = tc_gemm_run(q, stream);
            if (rc != MOE_OK) return rc;
        }
        const int64_t len = (int64_t)E * D;
        const int64_t nb = (len + 255) / 256;
        sum_rows_kernel<<<(unsigned)(nb < 4096 ? nb : 4096), 256, 0, stream>>>(part, 3 * S, len, dw);
        const int rc = launch_status();
        if (rc != MOE_OK) return rc;
    }
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_router_backward_workspace_size(int64_t T, int64_t D, int32_t E, moe_dtype dtype,
                                                     moe_router_layout layout) {
    if (T < 1 || D < 1 || E < 1) return 0;
    F32Gemm gx, gw;
    router_bwd_gemms(dtype, nullptr, T, D, D, nullptr, layout, E, nullptr, nullptr, nullptr, gx, gw);
    size_t total = router_bwd_layout(gx, gw, E).total;
    if (dtype == MOE_BF16 && moe::router_bwd_bf16_shape_ok(D, E)) {  // room for either path
        const size_t b = moe::router_bwd_bf16_layout(T, D, E).total;
        if (b > total) total = b;
    }
    return total;
}

extern "C" int moe_router_backward(moe_dtype dtype, const void* x, int64_t T, int64_t D, int64_t ldx,
                                   const void* w_router, moe_router_layout layout, int32_t E, const float* dlogits,
                                   float* dx_router, float* dw_router, float* db_router, int32_t* dev_status,
                                   void* workspace, size_t workspace_bytes, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(valid_dtype(dtype), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(layout == MOE_ROUTER_DE || layout == MOE_ROUTER_ED, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(x && w_router && dlogits && T >= 1 && D >= 1 && E >= 1 && ldx >= D, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(workspace_bytes >= moe_router_backward_workspace_size(T, D, E, dtype, layout) && workspace,
                MOE_ERR_WORKSPACE);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int rc;
    if (dtype == MOE_BF16 && router_bwd_bf16_shape_ok(D, E) && ldx % 8 == 0 && aligned16(x) && aligned16(w_router) &&
        T < (int64_t(1) << 31) / 3) {
        const RouterBwdBf16Ws lb = router_bwd_bf16_layout(T, D, E);
        if (dx_router || dw_router) {
            rc = router_backward_bf16(x, T, D, ldx, w_router, layout, E, dlogits, dx_router, dw_router, dev_status, ws,
                                      lb, stream);
            if (rc != MOE_OK) return rc;
        }
        if (db_router) {
            float* part = reinterpret_cast<float*>(ws + lb.colsum);
            const int64_t chunk = (T + kColChunks - 1) / kColChunks;
            const int chunks = (int)((T + chunk - 1) / chunk);
            column_sum_part_kernel<<<dim3((unsigned)((E + 31) / 32), (unsigned)chunks), 1024, 0, stream>>>(
                dlogits, T, E, chunk, part);
            rc = launch_status();
            if (rc != MOE_OK) return rc;
            sum_rows_kernel<<<(unsigned)((E + 255) / 256), 256, 0, stream>>>(part, chunks, E, db_router);
            return launch_status();
        }
        return MOE_OK;
    }
    F32Gemm gx, gw;
    router_bwd_gemms(dtype, x, T, D, ldx, w_router, layout, E, dlogits, dx_router, dw_router, gx, gw);
    const RouterBwdWs l = router_bwd_layout(gx, gw, E);
    if (dx_router) {
        rc = tf32x3_gemm_run(gx, ws, l.split, dev_status, stream);
        if (rc != MOE_OK) return rc;
    }
    if (dw_router) {
        float* part = reinterpret_cast<float*>(ws + l.split);
        if (gw.groups > 1) gw.C = part;
        rc = tf32x3_gemm_run(gw, ws, l.split, dev_status, stream);
        if (rc != MOE_OK) return rc;
        if (gw.groups > 1) {
            const int64_t len = gw.M * gw.N;
            const int64_t nb = (len + 255) / 256;
            sum_rows_kernel<<<(unsigned)(nb < 4096 ? nb : 4096), 256, 0, stream>>>(part, gw.groups, len, dw_router);
            rc = launch_status();
            if (rc != MOE_OK) return rc;
        }
    }
    if (db_router) {
        float* part = reinterpret_cast<float*>(ws + l.split + l.partials);
        const int64_t chunk = (T + kColChunks - 1) / kColChunks;
        const int chunks = (int)((T + chunk - 1) / chunk);
        column_sum_part_kernel<<<dim3((unsigned)((E + 31) / 32), (unsigned)chunks), 1024, 0, stream>>>(dlogits, T, E,
                                                                                                      chunk, part);
        rc = launch_status();
        if (rc != MOE_OK) return rc;
        sum_rows_kernel<<<(unsigned)((E + 255) / 256), 256, 0, stream>>>(part, chunks, E, db_router);
        return launch_status();
    }
    return MOE_OK;
}
