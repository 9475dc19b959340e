// fp32 FFMA GEMM: 128x128 block tile, K step 8, 256 threads with an 8x8
// register tile each, shared-memory double buffering.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "simt_gemm.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 128, BK = 8, PAD = 4, NT = 256;

template <bool AT, bool BT>
__global__ void __launch_bounds__(NT) sgemm_kernel(const SimtGemm g) {
    const int grp = blockIdx.z;
    int64_t Mg = g.M, Kg = g.K;
    if (g.rows_mode == 1) {
        const int64_t r = g.rows[grp];
        Mg = r < 0 ? 0 : (r < g.M ? r : g.M);
    } else if (g.rows_mode == 2) {
        const int64_t r = g.rows[grp];
        Kg = r < 0 ? 0 : (r < g.K ? r : g.K);
    }
    const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
    if (m0 >= Mg) return;
    const float* __restrict__ A = g.A + grp * g.a_group_stride;
    const float* __restrict__ B = g.B + grp * g.b_group_stride;
    float* __restrict__ C = g.C + grp * g.c_group_stride;
    const int64_t N = g.N, lda = g.lda, ldb = g.ldb;

    __shared__ __align__(16) float As[2][BK][BM + PAD];
    __shared__ __align__(16) float Bs[2][BK][BN + PAD];

    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    float ra[4], rb[4];
    auto load = [&](int64_t k0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int idx = tid + r * NT;
            int kk, mm;
            if (!AT) { kk = idx & 7; mm = idx >> 3; } else { mm = idx & 127; kk = idx >> 7; }
            const int64_t m = m0 + mm, k = k0 + kk;
            ra[r] = (m < Mg && k < Kg) ? (AT ? A[k * lda + m] : A[m * lda + k]) : 0.f;
            int nn;
            if (!BT) { nn = idx & 127; kk = idx >> 7; } else { kk = idx & 7; nn = idx >> 3; }
            const int64_t n = n0 + nn, kb = k0 + kk;
            rb[r] = (n < N && kb < Kg) ? (BT ? B[n * ldb + kb] : B[kb * ldb + n]) : 0.f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int idx = tid + r * NT;
            int kk, mm;
            if (!AT) { kk = idx & 7; mm = idx >> 3; } else { mm = idx & 127; kk = idx >> 7; }
            As[buf][kk][mm] = ra[r];
            int nn;
            if (!BT) { nn = idx & 127; kk = idx >> 7; } else { kk = idx & 7; nn = idx >> 3; }
            Bs[buf][kk][nn] = rb[r];
        }
    };

    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t k0 = 0; k0 < Kg; k0 += BK) {
        const bool has_next = k0 + BK < Kg;
        if (has_next) load(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (has_next) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }

    const float* bias = g.bias ? g.bias + grp * g.bias_group_stride : nullptr;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (m >= Mg) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
            if (n >= N) continue;
            float v = acc[i][j];
            float* dst = C + m * g.ldc + n;
            if (g.epilogue == SIMT_EPI_BIAS) {
                v += bias ? bias[n] : 0.f;
            } else if (g.epilogue == SIMT_EPI_BIAS_GELU) {
                v += bias ? bias[n] : 0.f;
                v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
            } else if (g.epilogue == SIMT_EPI_SILU_MUL) {
                v = (v / (1.0f + expf(-v))) * (*dst);
            }
            *dst = v;
        }
    }
}

}  // namespace

int simt_gemm_run(const SimtGemm& g, cudaStream_t stream) {
    MOE_REQUIRE(g.A && g.B && g.C && g.M >= 0 && g.N >= 0 && g.K >= 0 && g.groups >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(g.rows_mode == 0 || g.rows != nullptr, MOE_ERR_INVALID_ARG);
    if (g.M == 0 || g.N == 0) return MOE_OK;
    MOE_REQUIRE(g.groups <= 65535 && (g.M + BM - 1) / BM <= 65535, MOE_ERR_UNSUPPORTED);
    dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM), (unsigned)g.groups);
    if (!g.a_trans && !g.b_trans) sgemm_kernel<false, false><<<grid, NT, 0, stream>>>(g);
    else if (!g.a_trans && g.b_trans) sgemm_kernel<false, true><<<grid, NT, 0, stream>>>(g);
    else if (g.a_trans && !g.b_trans) sgemm_kernel<true, false><<<grid, NT, 0, stream>>>(g);
    else sgemm_kernel<true, true><<<grid, NT, 0, stream>>>(g);
    return launch_status();
}

}  // namespace moe
