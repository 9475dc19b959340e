// moe_backward: backward of the linear-expert layer with the kept mask fixed.
//   1. dgate / dlogits       one warp per token (row dots, quotient rule, aux term)
//   2. dybuf[e,c] = gate * dy[token]     token-major gather with scale
//   3. dW[e]   = dybuf_e^T xbuf_e        split-tf32 tensor-core GEMM, K = used[e] rows
//   4. dxbuf_e = dybuf_e W_e             split-tf32 tensor-core GEMM, M = used[e] rows
//   5. dx[t]   = [dy[t]] + sum_kept dxbuf[e, slot]   deterministic combine
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "f32_gemm.cuh"
#include "tc_tf32.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32)
    dgate_dlogits_kernel(const float* __restrict__ dy, int64_t Dout, const float* __restrict__ ybuf,
                         const float* __restrict__ logits, const int64_t* __restrict__ selected,
                         const float* __restrict__ gates, const int64_t* __restrict__ slot, int64_t T, int k, int E,
                         int64_t C, float aux_coef, float kn, const int32_t* __restrict__ counts,
                         float* __restrict__ dlogits, float* __restrict__ dgate, int32_t* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    if (t >= T) return;
    const float* dyr = dy + t * Dout;
    // dgate_j (all lanes end up with every dgate_j through the warp sums)
    float gdot = 0.f;
    float my_dg0 = 0.f, my_dg1 = 0.f;  // dgate for j = lane, lane + 32
    for (int j = 0; j < k; ++j) {
        const int64_t e = selected[t * k + j];
        const int64_t s = slot[t * k + j];
        float dg = 0.f;
        if (s >= 0) {
            if (e < 0 || e >= E || s >= C) {
                if (lane == 0) set_status(status, MOE_ERR_BAD_INDEX);
            } else {
                const float* yr = ybuf + (e * C + s) * Dout;
                float part = 0.f;
                for (int64_t n = lane; n < Dout; n += 32) part = fmaf(dyr[n], yr[n], part);
                dg = warp_sum(part);
            }
        }
        gdot = fmaf(gates[t * k + j], dg, gdot);
        if (j == lane) my_dg0 = dg;
        if (j == lane + 32) my_dg1 = dg;
    }
    if (lane < k) dgate[t * k + lane] = my_dg0;
    if (lane + 32 < k) dgate[t * k + lane + 32] = my_dg1;

    // aux term needs the softmax of the row
    float vmax = -INFINITY, cp = 0.f, inv = 0.f, scale = 0.f;
    const float* lr = logits + t * E;
    if (aux_coef != 0.f) {
        for (int e = lane; e < E; e += 32) vmax = fmaxf(vmax, lr[e]);
        vmax = warp_max(vmax);
        float den = 0.f;
        for (int e = lane; e < E; e += 32) den += expf(lr[e] - vmax);
        inv = 1.0f / warp_sum(den);
        float c = 0.f;
        for (int e = lane; e < E; e += 32) c += (float)counts[e] * (expf(lr[e] - vmax) * inv);
        cp = warp_sum(c);
        scale = aux_coef * (float)E / ((float)T * (float)T * kn);
    }
    // each lane owns columns e = lane + 32 m
    for (int e = lane; e < E; e += 32) {
        float v = 0.f;
        if (aux_coef != 0.f) {
            const float p = expf(lr[e] - vmax) * inv;
            v = scale * p * ((float)counts[e] - cp);
        }
        dlogits[t * E + e] = v;
    }
    __syncwarp();
    // quotient rule on the selected experts, in route-slot order
    for (int j = 0; j < k; ++j) {
        const float dg = __shfl_sync(0xffffffffu, j < 32 ? my_dg0 : my_dg1, j & 31);
        const int64_t e = selected[t * k + j];
        if (e < 0 || e >= E) continue;
        if ((int)(e & 31) == lane) {
            const float g = gates[t * k + j];
            dlogits[t * E + e] += g * (dg - gdot);
        }
        __syncwarp();
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace moe {
namespace {

// The two GEMMs' shapes (for the split-operand workspace).
size_t backward_split_bytes(int32_t E, int64_t C, int64_t D, int64_t Dout) {
    F32Gemm w{};  // dW: (Dout x D), K = C
    w.M = Dout;
    w.N = D;
    w.K = C;
    w.groups = E;
    F32Gemm x{};  // dxbuf: (C x D), K = Dout
    x.M = C;
    x.N = D;
    x.K = Dout;
    x.groups = E;
    const size_t a = tf32x3_workspace_size(w), b = tf32x3_workspace_size(x);
    return a > b ? a : b;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_backward_workspace_size(int32_t E, int64_t C, int64_t D, int64_t Dout) {
    if (E < 1 || C < 1) return 256;
    return align_up((size_t)E * C * Dout * 4, 256) + align_up((size_t)E * C * D * 4, 256) +
           backward_split_bytes(E, C, D, Dout);
}

extern "C" int moe_backward(moe_ffn_kind kind, moe_dtype dtype, const void* dy, const void* x, const float* logits,
                            const int64_t* selected, const float* gates, const int64_t* slot, const int32_t* used,
                            const int32_t* token_of_slot, const void* xbuf, const void* ybuf, const void* W,
                            int64_t T, int32_t k, int32_t E, int64_t C, int64_t D, int64_t Dout, int use_residual,
                            float aux_coef, int normalize_by_k, const int32_t* counts, void* dx, void* dW,
                            float* dlogits, float* dgate, int32_t* dev_status, void* workspace,
                            size_t workspace_bytes, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    (void)x;
    (void)token_of_slot;
    MOE_REQUIRE(kind == MOE_FFN_LINEAR && dtype == MOE_F32, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(dy && logits && selected && gates && slot && used && xbuf && ybuf && W && dx && dW && dlogits &&
                    dgate,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(T >= 1 && k >= 1 && k <= E && E >= 1 && C >= 0 && D >= 1 && Dout >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(k <= 64, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(!use_residual || Dout == D, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aux_coef == 0.f || counts != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(workspace && workspace_bytes >= moe_backward_workspace_size(E, C, D, Dout), MOE_ERR_WORKSPACE);
    const int64_t Cw = C > 0 ? C : 1;
    float* dybuf = static_cast<float*>(workspace);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* dxbuf = reinterpret_cast<float*>(ws + align_up((size_t)E * Cw * Dout * 4, 256));
    uint8_t* split = ws + align_up((size_t)E * Cw * Dout * 4, 256) + align_up((size_t)E * Cw * D * 4, 256);
    const size_t split_bytes = workspace_bytes - (size_t)(split - ws);

    const unsigned grid = (unsigned)((T + kWarps - 1) / kWarps);
    dgate_dlogits_kernel<<<grid, kWarps * 32, 0, stream>>>(
        static_cast<const float*>(dy), Dout, static_cast<const float*>(ybuf), logits, selected, gates, slot, T, k, E,
        C, aux_coef, normalize_by_k ? (float)k : 1.0f, counts, dlogits, dgate, dev_status);
    int rc = launch_status();
    if (rc != MOE_OK) return rc;

    if (C == 0) {
        // nothing kept: dW = 0, dx = [dy]
        MOE_CUDA_TRY(cudaMemsetAsync(dW, 0, (size_t)E * Dout * D * 4, stream));
        if (use_residual)
            MOE_CUDA_TRY(cudaMemcpyAsync(dx, dy, (size_t)T * D * 4, cudaMemcpyDeviceToDevice, stream));
        else
            MOE_CUDA_TRY(cudaMemsetAsync(dx, 0, (size_t)T * D * 4, stream));
        return MOE_OK;
    }

    rc = gather_rows(dy, Dout, T, k, selected, slot, E, C, gates, dybuf, Dout, MOE_F32, dev_status, stream);
    if (rc != MOE_OK) return rc;

    // dW[e] (Dout x D) = sum_c dybuf[e,c,:]^T xbuf[e,c,:]
    F32Gemm w{};
    w.A = dybuf;
    w.lda = Dout;
    w.a_trans = true;
    w.a_group_stride = C * Dout;
    w.B = static_cast<const float*>(xbuf);
    w.ldb = D;
    w.b_trans = false;
    w.b_group_stride = C * D;
    w.C = static_cast<float*>(dW);
    w.ldc = D;
    w.c_group_stride = Dout * D;
    w.M = Dout;
    w.N = D;
    w.K = C;
    w.groups = E;
    w.rows = used;
    w.rows_mode = 2;
    rc = tf32x3_gemm_run(w, split, split_bytes, dev_status, stream);
    if (rc != MOE_OK) return rc;

    // dxbuf[e] (rows x D) = dybuf[e] (rows x Dout) * W[e] (Dout x D)
    F32Gemm g{};
    g.A = dybuf;
    g.lda = Dout;
    g.a_group_stride = C * Dout;
    g.B = static_cast<const float*>(W);
    g.ldb = D;
    g.b_trans = false;
    g.b_group_stride = Dout * D;
    g.C = dxbuf;
    g.ldc = D;
    g.c_group_stride = C * D;
    g.M = C;
    g.N = D;
    g.K = Dout;
    g.groups = E;
    g.rows = used;
    g.rows_mode = 1;
    rc = tf32x3_gemm_run(g, split, split_bytes, dev_status, stream);
    if (rc != MOE_OK) return rc;

    return combine_rows(dxbuf, selected, slot, nullptr, MOE_F32, T, k, E, C, D, use_residual ? dy : nullptr, D, dx, D,
                        MOE_F32, dev_status, stream);
}
