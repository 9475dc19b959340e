// moe_backward: backward of the linear-expert layer with the kept mask fixed.
//   1. dgate / dlogits       one warp per token (row dots, quotient rule, aux term)
//   2. dybuf[e,c] = gate * dy[token]     token-major gather with scale
//   3. dW[e]   = dybuf_e^T xbuf_e        split-tf32 tensor-core GEMM, K = used[e] rows
//   4. dxbuf_e = dybuf_e W_e             split-tf32 tensor-core GEMM, M = used[e] rows
//   5. dx[t]   = [dy[t]] + sum_kept dxbuf[e, slot]   deterministic combine
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "tc_gemm.cuh"
#include "f32_gemm.cuh"
#include "tc_ptx.cuh"
#include "tc_tf32.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

// Dot products of rows of n elements, this lane's part: 16-byte vectors when
// VEC (n a multiple of the vector width, rows 16-byte aligned).
__device__ __forceinline__ float dot16(const uint4& a, const uint4& b, float acc, const float*) {
    acc = fmaf(__uint_as_float(a.x), __uint_as_float(b.x), acc);
    acc = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), acc);
    acc = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), acc);
    return fmaf(__uint_as_float(a.w), __uint_as_float(b.w), acc);
}
__device__ __forceinline__ float dot16(const uint4& a, const uint4& b, float acc, const __nv_bfloat16*) {
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[i]));
        const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[i]));
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
    }
    return acc;
}

// Two rows b0, b1 against one row a (a read once; a NULL row is skipped).
template <typename In, bool VEC>
__device__ __forceinline__ void row_dot_part2(const In* __restrict__ a, const In* __restrict__ b0,
                                              const In* __restrict__ b1, int64_t n, int lane, float& p0, float& p1) {
    p0 = 0.f;
    p1 = 0.f;
    if (VEC) {
        constexpr int EPV = 16 / sizeof(In);
        const int64_t nv = n / EPV;
        const uint4* va = reinterpret_cast<const uint4*>(a);
        const uint4* v0 = reinterpret_cast<const uint4*>(b0);
        const uint4* v1 = reinterpret_cast<const uint4*>(b1);
        for (int64_t v = lane; v < nv; v += 32) {
            const uint4 x = va[v];
            if (b0) p0 = dot16(x, v0[v], p0, a);
            if (b1) p1 = dot16(x, v1[v], p1, a);
        }
    } else {
        for (int64_t i = lane; i < n; i += 32) {
            const float x = to_f32(a[i]);
            if (b0) p0 = fmaf(x, to_f32(b0[i]), p0);
            if (b1) p1 = fmaf(x, to_f32(b1[i]), p1);
        }
    }
}

template <typename In, bool VEC>
__global__ void __launch_bounds__(kWarps * 32)
    dgate_dlogits_kernel(const In* __restrict__ dy, int64_t Dout, const In* __restrict__ ybuf,
                         const float* __restrict__ logits, const int64_t* __restrict__ selected,
                         const float* __restrict__ gates, const int64_t* __restrict__ slot, int64_t T, int k, int E,
                         int64_t C, float aux_coef, float kn, const int32_t* __restrict__ counts,
                         float* __restrict__ dlogits, float* __restrict__ dgate, int32_t* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    if (t >= T) return;
    const In* dyr = dy + t * Dout;
    // dgate_j (all lanes end up with every dgate_j through the warp sums)
    float gdot = 0.f;
    float my_dg0 = 0.f, my_dg1 = 0.f;  // dgate for j = lane, lane + 32
    // two assignments at a time: the dy row is read once for both, and both rows' loads are in flight
    for (int j = 0; j < k; j += 2) {
        const In* yr[2] = {nullptr, nullptr};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (j + u >= k) break;
            const int64_t e = selected[t * k + j + u];
            const int64_t s = slot[t * k + j + u];
            if (s >= 0) {
                if (e < 0 || e >= E || s >= C) {
                    if (lane == 0) set_status(status, MOE_ERR_BAD_INDEX);
                } else {
                    yr[u] = ybuf + (e * C + s) * Dout;
                }
            }
        }
        float p0, p1;
        row_dot_part2<In, VEC>(dyr, yr[0], yr[1], Dout, lane, p0, p1);
        const float dg0 = yr[0] ? warp_sum(p0) : 0.f;
        const float dg1 = yr[1] ? warp_sum(p1) : 0.f;
        gdot = fmaf(gates[t * k + j], dg0, gdot);
        if (j == lane) my_dg0 = dg0;
        if (j == lane + 32) my_dg1 = dg0;
        if (j + 1 < k) {
            gdot = fmaf(gates[t * k + j + 1], dg1, gdot);
            if (j + 1 == lane) my_dg0 = dg1;
            if (j + 1 == lane + 32) my_dg1 = dg1;
        }
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

template <typename In>
void launch_dgate(unsigned grid, cudaStream_t stream, const In* dy, int64_t Dout, const In* ybuf,
                  const float* logits, const int64_t* selected, const float* gates, const int64_t* slot, int64_t T,
                  int k, int E, int64_t C, float aux_coef, float kn, const int32_t* counts, float* dlogits,
                  float* dgate, int32_t* status) {
    constexpr int EPV = 16 / sizeof(In);
    const bool vec = Dout % EPV == 0 && aligned16(dy) && (ybuf == nullptr || aligned16(ybuf));
    if (vec)
        dgate_dlogits_kernel<In, true><<<grid, kWarps * 32, 0, stream>>>(dy, Dout, ybuf, logits, selected, gates, slot,
                                                                        T, k, E, C, aux_coef, kn, counts, dlogits,
                                                                        dgate, status);
    else
        dgate_dlogits_kernel<In, false><<<grid, kWarps * 32, 0, stream>>>(dy, Dout, ybuf, logits, selected, gates,
                                                                         slot, T, k, E, C, aux_coef, kn, counts,
                                                                         dlogits, dgate, status);
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
    launch_dgate<float>(grid, stream, static_cast<const float*>(dy), Dout, static_cast<const float*>(ybuf), logits,
                        selected, gates, slot, T, k, E, C, aux_coef, normalize_by_k ? (float)k : 1.0f, counts, dlogits,
                        dgate, dev_status);
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

// ---------------------------------------------------------------------------
// moe_backward_swiglu: bf16 SwiGLU experts, the kept mask held constant.
//   1. dgate / dlogits                       as above, on bf16 rows
//   2. dybuf[e,c] = gate * dy[token]         scaled gather (bf16)
//   3. [a | b] = xbuf [Wg; Wu]^T             one tensor-core GEMM (both weights), fp32 out,
//                                            unless the forward saved them (bf16)
//   4. dh = dybuf Wd                         tensor-core GEMM, fp32 out
//   5. h, da, db from (a, b, dh)             elementwise (silu and its derivative)
//   6. dWd = dybuf^T h, dWg = da^T xbuf, dWu = db^T xbuf
//                                            tensor-core GEMMs over each expert's kept
//                                            tokens, fp32 out
//   7. dxbuf = [da | db] [Wg; Wu]            tensor-core GEMM, bf16 out
//   8. dx[t] = [dy[t]] + sum_kept dxbuf[e, slot]
// All products run on the tcgen05 kernel.  With H and F multiples of 64 every
// operand is read in place (the weights and, for step 6, both token-major
// operands as MN-major operands); otherwise the operands that need another
// major order are transposed first (zero past used[e] for the token-major ones).
// ---------------------------------------------------------------------------
namespace moe {
namespace {

// dst[g][c][r] = r < valid[g] ? src[g][r][c] : 0   for r < Rp, c < Cc
// (valid = NULL: every r < R is valid).  bf16; 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256)
    transpose_valid_kernel(const __nv_bfloat16* __restrict__ src, int64_t lds, int64_t sgs, int64_t R, int64_t Cc,
                           const int32_t* __restrict__ valid, int64_t Rp, __nv_bfloat16* __restrict__ dst,
                           int64_t ldd, int64_t dgs) {
    __shared__ __nv_bfloat16 tile[32][34];
    const int g = blockIdx.z;
    int64_t Rv = R;
    if (valid) {
        const int64_t v = valid[g];
        Rv = v < 0 ? 0 : (v < R ? v : R);
    }
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    const __nv_bfloat16* s = src + g * sgs;
    __nv_bfloat16* d = dst + g * dgs;
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int64_t r = r0 + i, c = c0 + threadIdx.x;
        tile[i][threadIdx.x] = (r < Rv && c < Cc) ? s[r * lds + c] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int64_t c = c0 + i, r = r0 + threadIdx.x;
        if (c < Cc && r < Rp) d[c * ldd + r] = tile[threadIdx.x][i];
    }
}

// The same transpose on 64 x 64 tiles moving 16-byte vectors on both sides
// (with `valid`, 64-wide row blocks wholly past the valid rows, other than the
// first, are left unwritten: the GEMMs that read them stop at the valid count)
// (needs 16-byte aligned bases, strides that are multiples of 8 elements,
// Cc and Rp multiples of 8).  Tile rows are 66 elements wide (33 words), so
// the column reads of the second phase hit at most two lanes per bank.
constexpr int kTT = 64;
__global__ void __launch_bounds__(256)
    transpose_valid_v8_kernel(const __nv_bfloat16* __restrict__ src, int64_t lds, int64_t sgs, int64_t R, int64_t Cc,
                              const int32_t* __restrict__ valid, int64_t Rp, __nv_bfloat16* __restrict__ dst,
                              int64_t ldd, int64_t dgs) {
    __shared__ uint16_t tile[kTT][kTT + 2];
    const int g = blockIdx.z;
    int64_t Rv = R;
    if (valid) {
        const int64_t v = valid[g];
        Rv = v < 0 ? 0 : (v < R ? v : R);
    }
    const int64_t r0 = (int64_t)blockIdx.y * kTT, c0 = (int64_t)blockIdx.x * kTT;
    // with a valid count, only the 64-wide blocks a K-limited product reads are
    // needed: those up to the one holding row Rv - 1 (at least the first)
    if (valid && r0 >= kTT && r0 >= Rv) return;
    const __nv_bfloat16* s = src + g * sgs;
    __nv_bfloat16* d = dst + g * dgs;
    const int q = threadIdx.x & 7, rr = threadIdx.x >> 3;  // 8-element chunk, row within a 32-row half
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int64_t r = r0 + rr + 32 * i, c = c0 + 8 * q;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < Rv && c < Cc) v = *reinterpret_cast<const uint4*>(s + r * lds + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            tile[rr + 32 * i][8 * q + 2 * j] = (uint16_t)(w[j] & 0xFFFFu);
            tile[rr + 32 * i][8 * q + 2 * j + 1] = (uint16_t)(w[j] >> 16);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int64_t c = c0 + rr + 32 * i, r = r0 + 8 * q;
        if (c < Cc && r < Rp) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = (uint32_t)tile[8 * q + 2 * j][rr + 32 * i] | ((uint32_t)tile[8 * q + 2 * j + 1][rr + 32 * i] << 16);
            *reinterpret_cast<uint4*>(d + c * ldd + r) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

int transpose_valid(const __nv_bfloat16* src, int64_t lds, int64_t sgs, int G, int64_t R, int64_t Cc,
                    const int32_t* valid, int64_t Rp, __nv_bfloat16* dst, int64_t ldd, int64_t dgs,
                    cudaStream_t stream) {
    MOE_REQUIRE(G <= 65535 && (Rp + 31) / 32 <= 65535, MOE_ERR_UNSUPPORTED);
    const bool v8 = aligned16(src) && aligned16(dst) && lds % 8 == 0 && sgs % 8 == 0 && ldd % 8 == 0 &&
                    dgs % 8 == 0 && Cc % 8 == 0 && Rp % 8 == 0;
    if (v8) {
        const dim3 grid((unsigned)((Cc + kTT - 1) / kTT), (unsigned)((Rp + kTT - 1) / kTT), (unsigned)G);
        transpose_valid_v8_kernel<<<grid, 256, 0, stream>>>(src, lds, sgs, R, Cc, valid, Rp, dst, ldd, dgs);
    } else {
        const dim3 grid((unsigned)((Cc + 31) / 32), (unsigned)((Rp + 31) / 32), (unsigned)G), block(32, 8);
        transpose_valid_kernel<<<grid, block, 0, stream>>>(src, lds, sgs, R, Cc, valid, Rp, dst, ldd, dgs);
    }
    return launch_status();
}

// h, da, db from a, b (ab rows: [a | b], fp32, or bf16 when saved by the forward) and dh
// (fp32), for c < used[e]:
//   s = sigmoid(a), h = a s b, da = dh b s (1 + a (1 - s)), db = dh a s.
// Eight consecutive f per thread (F a multiple of 8): vector loads, 16-byte bf16 stores.
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 x = reinterpret_cast<const float4*>(p)[0], y = reinterpret_cast<const float4*>(p)[1];
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

template <typename AB>
__global__ void swiglu_bwd_elem_kernel(const AB* __restrict__ ab, const float* __restrict__ dh,
                                       const int32_t* __restrict__ used, int64_t C, int64_t F,
                                       __nv_bfloat16* __restrict__ h, __nv_bfloat16* __restrict__ dab) {
    const int e = blockIdx.y;
    const int64_t u = used[e] < 0 ? 0 : (used[e] < C ? used[e] : C);
    const int64_t F8 = F / 8;
    const int64_t n = u * F8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = i / F8, f = (i - c * F8) * 8;
        const int64_t row = (int64_t)e * C + c;
        float av[8], bv[8], gv[8];
        load8(ab + row * 2 * F + f, av);
        load8(ab + row * 2 * F + F + f, bv);
        load8(dh + row * F + f, gv);
        uint32_t ph[4], pda[4], pdb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float hv[2], dav[2], dbv[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const float a = av[2 * j + m], b = bv[2 * j + m], g = gv[2 * j + m];
                const float s = 1.0f / (1.0f + expf(-a));
                hv[m] = a * s * b;
                dav[m] = g * b * s * (1.0f + a * (1.0f - s));
                dbv[m] = g * a * s;
            }
            ph[j] = tc::pack_bf16x2(hv[0], hv[1]);
            pda[j] = tc::pack_bf16x2(dav[0], dav[1]);
            pdb[j] = tc::pack_bf16x2(dbv[0], dbv[1]);
        }
        *reinterpret_cast<uint4*>(h + row * F + f) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(dab + row * 2 * F + f) = make_uint4(pda[0], pda[1], pda[2], pda[3]);
        *reinterpret_cast<uint4*>(dab + row * 2 * F + F + f) = make_uint4(pdb[0], pdb[1], pdb[2], pdb[3]);
    }
}

// Grouped bf16 GEMM out[g] (M x N, fp32 or bf16) = A[g] (M x K) B[g]^T, K-major operands.
int gemm(const void* a, int64_t lda, int64_t a_rows_total, int64_t a_rows_per_group, const void* b, int64_t ldb,
         int64_t b_rows_total, int64_t b_rows_per_group, int G, int64_t M, int64_t N, int64_t K, const int32_t* rows,
         void* out, int64_t ldo, int64_t out_rows_per_group, int epilogue, int32_t* status, cudaStream_t stream,
         const int32_t* k_rows = nullptr) {
    TcGemmProblem p{};
    p.a = a;
    p.lda = lda;
    p.a_rows_total = a_rows_total;
    p.a_rows_per_group = a_rows_per_group;
    p.b = b;
    p.ldb = ldb;
    p.b_rows_total = b_rows_total;
    p.b_rows_per_group = b_rows_per_group;
    p.G = G;
    p.M = M;
    p.N = N;
    p.K = K;
    p.rows = rows;
    p.k_rows = k_rows;
    p.out = out;
    p.ldo = ldo;
    p.out_rows_per_group = out_rows_per_group;
    p.epilogue = epilogue;
    p.status = status;
    return tc_gemm_run(p, stream);
}

struct SwigluBwdWs {
    size_t dybuf, ab, dh, h, dab, wdT, wguT, dybufT, hT, dabT, xbufT, dxbuf, total;
    int64_t Cp;
};

SwigluBwdWs swiglu_bwd_layout(int32_t E, int64_t C, int64_t H, int64_t F) {
    SwigluBwdWs w{};
    w.Cp = (C + 7) / 8 * 8;  // token count padded for 16-byte TMA rows
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align_up(bytes, 1024);
        return o;
    };
    w.dybuf = take((size_t)E * C * H * 2);
    w.ab = take((size_t)E * C * 2 * F * 4);
    w.dh = take((size_t)E * C * F * 4);
    w.h = take((size_t)E * C * F * 2);
    w.dab = take((size_t)E * C * 2 * F * 2);
    const bool mn = H % 64 == 0 && F % 64 == 0;  // weights read in place (MN-major): no transposed copies
    w.wdT = take(mn ? 0 : (size_t)E * F * H * 2);
    w.wguT = take(mn ? 0 : (size_t)E * H * 2 * F * 2);
    // token-transposed operands of the weight gradients (not needed when both operands are read MN-major)
    w.dybufT = take(mn ? 0 : (size_t)E * H * w.Cp * 2);
    w.hT = take(mn ? 0 : (size_t)E * F * w.Cp * 2);
    w.dabT = take(mn ? 0 : (size_t)E * 2 * F * w.Cp * 2);
    w.xbufT = take(mn ? 0 : (size_t)E * H * w.Cp * 2);
    w.dxbuf = take((size_t)E * C * H * 2);
    w.total = off;
    return w;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_backward_swiglu_workspace_size(int32_t E, int64_t C, int64_t H, int64_t F) {
    if (E < 1 || C < 1 || H < 1 || F < 1) return 256;
    return swiglu_bwd_layout(E, C, H, F).total;
}

extern "C" int moe_backward_swiglu(moe_dtype dtype, const void* dy, const float* logits, const int64_t* selected,
                                   const float* gates, const int64_t* slot, const int32_t* used, const void* xbuf,
                                   const void* ybuf, const void* saved_ab, const void* w_gate, const void* w_up, const void* w_down,
                                   int64_t T, int32_t k, int32_t E, int64_t C, int64_t H, int64_t F, int use_residual,
                                   float aux_coef, int normalize_by_k, const int32_t* counts, void* dx,
                                   float* dw_gate, float* dw_up, float* dw_down, float* dlogits, float* dgate,
                                   int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                   moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    using bf16 = __nv_bfloat16;
    MOE_REQUIRE(dtype == MOE_BF16, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(dy && logits && selected && gates && slot && used && dx && dw_gate && dw_up && dw_down && dlogits &&
                    dgate,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(C == 0 || (xbuf && ybuf && w_gate && w_up && w_down), MOE_ERR_INVALID_ARG);  // unread when C == 0
    MOE_REQUIRE(T >= 1 && k >= 1 && k <= E && E >= 1 && C >= 0 && H >= 1 && F >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(k <= 64 && H % 8 == 0 && F % 8 == 0, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(aux_coef == 0.f || counts != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(workspace && workspace_bytes >= moe_backward_swiglu_workspace_size(E, C, H, F), MOE_ERR_WORKSPACE);

    const unsigned grid = (unsigned)((T + kWarps - 1) / kWarps);
    launch_dgate<bf16>(grid, stream, static_cast<const bf16*>(dy), H, static_cast<const bf16*>(ybuf), logits, selected,
                       gates, slot, T, k, E, C, aux_coef, normalize_by_k ? (float)k : 1.0f, counts, dlogits, dgate,
                       dev_status);
    int rc = launch_status();
    if (rc != MOE_OK) return rc;

    if (C == 0) {  // nothing kept: no expert gradient
        MOE_CUDA_TRY(cudaMemsetAsync(dw_gate, 0, (size_t)E * F * H * 4, stream));
        MOE_CUDA_TRY(cudaMemsetAsync(dw_up, 0, (size_t)E * F * H * 4, stream));
        MOE_CUDA_TRY(cudaMemsetAsync(dw_down, 0, (size_t)E * H * F * 4, stream));
        if (use_residual)
            MOE_CUDA_TRY(cudaMemcpyAsync(dx, dy, (size_t)T * H * 2, cudaMemcpyDeviceToDevice, stream));
        else
            MOE_CUDA_TRY(cudaMemsetAsync(dx, 0, (size_t)T * H * 2, stream));
        return MOE_OK;
    }

    const SwigluBwdWs l = swiglu_bwd_layout(E, C, H, F);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    bf16* dybuf = reinterpret_cast<bf16*>(ws + l.dybuf);
    float* ab = reinterpret_cast<float*>(ws + l.ab);
    float* dh = reinterpret_cast<float*>(ws + l.dh);
    bf16* h = reinterpret_cast<bf16*>(ws + l.h);
    bf16* dab = reinterpret_cast<bf16*>(ws + l.dab);
    bf16* wdT = reinterpret_cast<bf16*>(ws + l.wdT);
    bf16* wguT = reinterpret_cast<bf16*>(ws + l.wguT);
    bf16* dybufT = reinterpret_cast<bf16*>(ws + l.dybufT);
    bf16* hT = reinterpret_cast<bf16*>(ws + l.hT);
    bf16* dabT = reinterpret_cast<bf16*>(ws + l.dabT);
    bf16* xbufT = reinterpret_cast<bf16*>(ws + l.xbufT);
    bf16* dxbuf = reinterpret_cast<bf16*>(ws + l.dxbuf);
    const int64_t Cp = l.Cp, F2 = 2 * F;
    const bf16* xb = static_cast<const bf16*>(xbuf);

    // 2. dybuf[e,c] = gate * dy[token]
    rc = gather_rows(dy, H, T, k, selected, slot, E, C, gates, dybuf, H, MOE_BF16, dev_status, stream);
    if (rc != MOE_OK) return rc;
    // 3. [a | b] = xbuf [Wg; Wu]^T  (fp32), both weights in one pass over xbuf, unless the
    //    forward saved them (bf16, moe_expert_ffn_save)
    if (saved_ab == nullptr) {
        TcGemmProblem p{};
        p.a = xbuf;
        p.lda = H;
        p.a_rows_total = (int64_t)E * C;
        p.a_rows_per_group = C;
        p.b = w_gate;
        p.b2 = w_up;
        p.ldb = H;
        p.b_rows_total = (int64_t)E * F;
        p.b_rows_per_group = F;
        p.G = E;
        p.M = C;
        p.N = F;
        p.K = H;
        p.rows = used;
        p.out = ab;
        p.ldo = F2;
        p.out_rows_per_group = C;
        p.epilogue = TC_EPI_F32_DUAL;
        p.status = dev_status;
        rc = tc_gemm_run(p, stream);
        if (rc != MOE_OK) return rc;
    }
    // With H and F multiples of 64 the weights are read in their own layout as MN-major
    // operands; otherwise transposed copies feed the K-major form.
    const bool mn = H % 64 == 0 && F % 64 == 0;
    // 4. dh = dybuf Wd: B(k = h, n = f) = Wd[e][h][f].  With the forward's bf16 [a | b] at hand the
    //    GEMM's epilogue also does step 5 (h, da, db from the dh accumulator), so dh never reaches HBM.
    const bool fused_elem = mn && saved_ab != nullptr;
    if (mn) {
        TcGemmProblem p{};
        p.a = dybuf;
        p.lda = H;
        p.a_rows_total = (int64_t)E * C;
        p.a_rows_per_group = C;
        p.b = w_down;
        p.ldb = F;
        p.b_rows_total = (int64_t)E * H;
        p.b_rows_per_group = H;
        p.b_mn_major = true;
        p.G = E;
        p.M = C;
        p.N = F;
        p.K = H;
        p.rows = used;
        if (fused_elem) {
            p.out = dab;
            p.ldo = F2;
            p.ab = saved_ab;
            p.h = h;
            p.epilogue = TC_EPI_SWIGLU_BWD;
        } else {
            p.out = dh;
            p.ldo = F;
            p.epilogue = TC_EPI_F32;
        }
        p.out_rows_per_group = C;
        p.status = dev_status;
        rc = tc_gemm_run(p, stream);
    } else {
        rc = transpose_valid(static_cast<const bf16*>(w_down), F, H * F, E, H, F, nullptr, H, wdT, H, F * H, stream);
        if (rc != MOE_OK) return rc;
        rc = gemm(dybuf, H, (int64_t)E * C, C, wdT, H, (int64_t)E * F, F, E, C, F, H, used, dh, F, C, TC_EPI_F32,
                  dev_status, stream);
    }
    if (rc != MOE_OK) return rc;
    // 5. h, da, db
    if (!fused_elem) {
        const int64_t nb = (C * (F / 8) + 255) / 256;
        const dim3 g2((unsigned)(nb < 1024 ? nb : 1024), (unsigned)E);
        MOE_REQUIRE(E <= 65535, MOE_ERR_UNSUPPORTED);
        if (saved_ab)
            swiglu_bwd_elem_kernel<bf16><<<g2, 256, 0, stream>>>(static_cast<const bf16*>(saved_ab), dh, used, C, F,
                                                                 h, dab);
        else
            swiglu_bwd_elem_kernel<float><<<g2, 256, 0, stream>>>(ab, dh, used, C, F, h, dab);
        rc = launch_status();
        if (rc != MOE_OK) return rc;
    }
    // 6. weight gradients over the token index, K = the expert's kept tokens.  With H and F multiples
    //    of 64 both operands are read in place with the token on their rows (MN-major A and B; the
    //    GEMM clears the rows past used[e] of an expert's last K block); otherwise from transposed
    //    copies that are zero past used[e].
    if (mn) {
        auto wgrad = [&](const void* a, int64_t lda, int64_t M, const void* b, int64_t ldb, int64_t N, float* out,
                         float* out2 = nullptr, int64_t m_split = 0) {
            TcGemmProblem p{};
            p.a = a;
            p.lda = lda;
            p.a_rows_total = (int64_t)E * C;
            p.a_rows_per_group = C;
            p.a_mn_major = true;
            p.b = b;
            p.ldb = ldb;
            p.b_rows_total = (int64_t)E * C;
            p.b_rows_per_group = C;
            p.b_mn_major = true;
            p.G = E;
            p.M = M;
            p.N = N;
            p.K = C;
            p.k_rows = used;
            p.out = out;
            p.out2 = out2;
            p.m_split = m_split;
            p.ldo = N;
            p.out_rows_per_group = m_split > 0 ? m_split : M;
            p.epilogue = TC_EPI_F32;
            p.status = dev_status;
            return tc_gemm_run(p, stream);
        };
        if ((rc = wgrad(dybuf, H, H, h, F, F, dw_down)) != MOE_OK) return rc;  // dWd[e] (H, F) = dybuf^T h
        if (F % 128 == 0) {
            // [dWg; dWu][e] (2F, H) = [da | db]^T x in one GEMM: each x tile is read from HBM once for
            // both gradients (the tiles of an expert run back to back, its x stays in L2); rows >= F go to dWu
            if ((rc = wgrad(dab, F2, F2, xb, H, H, dw_gate, dw_up, F)) != MOE_OK) return rc;
        } else {
            if ((rc = wgrad(dab, F2, F, xb, H, H, dw_gate)) != MOE_OK) return rc;  // dWg[e] (F, H) = da^T x
            if ((rc = wgrad(dab + F, F2, F, xb, H, H, dw_up)) != MOE_OK) return rc;  // dWu[e] (F, H) = db^T x
        }
    } else {
        rc = transpose_valid(dybuf, H, C * H, E, C, H, used, Cp, dybufT, Cp, H * Cp, stream);
        if (rc != MOE_OK) return rc;
        rc = transpose_valid(h, F, C * F, E, C, F, used, Cp, hT, Cp, F * Cp, stream);
        if (rc != MOE_OK) return rc;
        rc = transpose_valid(dab, F2, C * F2, E, C, F2, used, Cp, dabT, Cp, F2 * Cp, stream);
        if (rc != MOE_OK) return rc;
        rc = transpose_valid(xb, H, C * H, E, C, H, used, Cp, xbufT, Cp, H * Cp, stream);
        if (rc != MOE_OK) return rc;
        // K = the expert's kept tokens only (the transposed operands are zero past used[e])
        rc = gemm(dybufT, Cp, (int64_t)E * H, H, hT, Cp, (int64_t)E * F, F, E, H, F, Cp, nullptr, dw_down, F, H,
                  TC_EPI_F32, dev_status, stream, used);
        if (rc != MOE_OK) return rc;
        rc = gemm(dabT, Cp, (int64_t)E * F2, F2, xbufT, Cp, (int64_t)E * H, H, E, F, H, Cp, nullptr, dw_gate, H, F,
                  TC_EPI_F32, dev_status, stream, used);
        if (rc != MOE_OK) return rc;
        rc = gemm(dabT + F * Cp, Cp, (int64_t)E * F2 - F, F2, xbufT, Cp, (int64_t)E * H, H, E, F, H, Cp, nullptr, dw_up,
                  H, F, TC_EPI_F32, dev_status, stream, used);
        if (rc != MOE_OK) return rc;
    }
    // 7. dxbuf = [da | db] [Wg; Wu]: B(k, n = h) = Wg[e][k][h] for k < F, Wu[e][k - F][h] after
    if (mn) {
        TcGemmProblem p{};
        p.a = dab;
        p.lda = F2;
        p.a_rows_total = (int64_t)E * C;
        p.a_rows_per_group = C;
        p.b = w_gate;
        p.b2 = w_up;
        p.k_split = F;
        p.ldb = H;
        p.b_rows_total = (int64_t)E * F;
        p.b_rows_per_group = F;
        p.b_mn_major = true;
        p.G = E;
        p.M = C;
        p.N = H;
        p.K = F2;
        p.rows = used;
        p.out = dxbuf;
        p.ldo = H;
        p.out_rows_per_group = C;
        p.epilogue = TC_EPI_BF16;
        p.status = dev_status;
        rc = tc_gemm_run(p, stream);
    } else {
        rc = transpose_valid(static_cast<const bf16*>(w_gate), H, F * H, E, F, H, nullptr, F, wguT, F2, H * F2,
                             stream);
        if (rc != MOE_OK) return rc;
        rc = transpose_valid(static_cast<const bf16*>(w_up), H, F * H, E, F, H, nullptr, F, wguT + F, F2, H * F2,
                             stream);
        if (rc != MOE_OK) return rc;
        rc = gemm(dab, F2, (int64_t)E * C, C, wguT, F2, (int64_t)E * H, H, E, C, H, F2, used, dxbuf, H, C,
                  TC_EPI_BF16, dev_status, stream);
    }
    if (rc != MOE_OK) return rc;
    // 8. dx
    return combine_rows(dxbuf, selected, slot, nullptr, MOE_F32, T, k, E, C, H, use_residual ? dy : nullptr, H, dx,
                        H, MOE_BF16, dev_status, stream);
}

// ---------------------------------------------------------------------------
// moe_backward_gelu: fp32 GELU-MLP experts (fc2(gelu(fc1 x)), both layers with
// bias), the kept mask held constant.
//   1. dgate / dlogits                       as above
//   2. dybuf[e,c] = gate * dy[token]         scaled gather
//   3. z  = xbuf W1^T + b1                   split-tf32 GEMM, bias epilogue
//   4. dh = dybuf W2                         split-tf32 GEMM
//   5. h = gelu(z), dz = dh * gelu'(z)       elementwise, in place over z and dh
//   6. dW2 = dybuf^T h,  dW1 = dz^T xbuf     split-tf32 GEMMs, K = used[e] tokens
//   7. db2 = column sums of dybuf, db1 = column sums of dz (c < used[e], fixed order)
//   8. dxbuf = dz W1                         split-tf32 GEMM
//   9. dx[t] = [dy[t]] + sum_kept dxbuf[e, slot]
// ---------------------------------------------------------------------------
namespace moe {
namespace {

// In place over the first used[e] rows of expert e:
//   z  <- gelu(z)                       = z Phi(z)
//   dh <- dh * gelu'(z),  gelu'(z)      = Phi(z) + z phi(z)
// with Phi the standard normal CDF (through erff) and phi its density.
__global__ void gelu_bwd_elem_kernel(float* __restrict__ z, float* __restrict__ dh, const int32_t* __restrict__ used,
                                     int64_t C, int64_t F) {
    const int e = blockIdx.y;
    const int64_t u = used[e] < 0 ? 0 : (used[e] < C ? used[e] : C);
    const int64_t n = u * F;
    float* ze = z + (int64_t)e * C * F;
    float* de = dh + (int64_t)e * C * F;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = ze[i];
        const float cdf = 0.5f * (1.0f + erff(v * 0.70710678118654752f));
        const float pdf = 0.39894228040143268f * expf(-0.5f * v * v);
        ze[i] = v * cdf;
        de[i] *= cdf + v * pdf;
    }
}

// out[g][n] = sum_{r < valid[g]} src[g][r][n], r ascending (one thread per column).
__global__ void group_column_sum_kernel(const float* __restrict__ src, int64_t R, int64_t N,
                                        const int32_t* __restrict__ valid, float* __restrict__ out) {
    const int g = blockIdx.y;
    const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int64_t u = valid[g] < 0 ? 0 : (valid[g] < R ? valid[g] : R);
    const float* s = src + (int64_t)g * R * N + n;
    float acc = 0.f;
    for (int64_t r = 0; r < u; ++r) acc += s[r * N];
    out[(int64_t)g * N + n] = acc;
}

struct GeluBwdWs {
    size_t dybuf, z, dh, dxbuf, split, total;
};

// The five split-tf32 GEMMs (operand pointers filled in by the caller).
void gelu_bwd_shapes(int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout, F32Gemm (&s)[5]) {
    for (auto& q : s) {
        q = F32Gemm{};
        q.groups = E;
    }
    // 0: z (C x F) = xbuf (C x D) . W1^T, W1 (F, D)
    s[0].lda = D; s[0].a_group_stride = C * D;
    s[0].ldb = D; s[0].b_trans = true; s[0].b_group_stride = F * D;
    s[0].ldc = F; s[0].c_group_stride = C * F;
    s[0].M = C; s[0].N = F; s[0].K = D; s[0].rows_mode = 1;
    s[0].bias_group_stride = F; s[0].epilogue = F32_EPI_BIAS;
    // 1: dh (C x F) = dybuf (C x Dout) . W2, W2 (Dout, F)
    s[1].lda = Dout; s[1].a_group_stride = C * Dout;
    s[1].ldb = F; s[1].b_group_stride = Dout * F;
    s[1].ldc = F; s[1].c_group_stride = C * F;
    s[1].M = C; s[1].N = F; s[1].K = Dout; s[1].rows_mode = 1;
    // 2: dW2 (Dout x F) = dybuf^T (Dout x C) . h (C x F)
    s[2].lda = Dout; s[2].a_trans = true; s[2].a_group_stride = C * Dout;
    s[2].ldb = F; s[2].b_group_stride = C * F;
    s[2].ldc = F; s[2].c_group_stride = Dout * F;
    s[2].M = Dout; s[2].N = F; s[2].K = C; s[2].rows_mode = 2;
    // 3: dW1 (F x D) = dz^T (F x C) . xbuf (C x D)
    s[3].lda = F; s[3].a_trans = true; s[3].a_group_stride = C * F;
    s[3].ldb = D; s[3].b_group_stride = C * D;
    s[3].ldc = D; s[3].c_group_stride = F * D;
    s[3].M = F; s[3].N = D; s[3].K = C; s[3].rows_mode = 2;
    // 4: dxbuf (C x D) = dz (C x F) . W1 (F x D)
    s[4].lda = F; s[4].a_group_stride = C * F;
    s[4].ldb = D; s[4].b_group_stride = F * D;
    s[4].ldc = D; s[4].c_group_stride = C * D;
    s[4].M = C; s[4].N = D; s[4].K = F; s[4].rows_mode = 1;
}

GeluBwdWs gelu_bwd_layout(int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout) {
    GeluBwdWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align_up(bytes, 1024);
        return o;
    };
    w.dybuf = take((size_t)E * C * Dout * 4);
    w.z = take((size_t)E * C * F * 4);
    w.dh = take((size_t)E * C * F * 4);
    w.dxbuf = take((size_t)E * C * D * 4);
    F32Gemm s[5];
    gelu_bwd_shapes(E, C, D, F, Dout, s);
    size_t split = 0;
    for (const auto& q : s) {
        const size_t b = tf32x3_workspace_size(q);
        split = b > split ? b : split;
    }
    w.split = take(split);
    w.total = off;
    return w;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_backward_gelu_workspace_size(int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout) {
    if (E < 1 || C < 1 || D < 1 || F < 1 || Dout < 1) return 256;
    return gelu_bwd_layout(E, C, D, F, Dout).total;
}

extern "C" int moe_backward_gelu(moe_dtype dtype, const void* dy, const float* logits, const int64_t* selected,
                                 const float* gates, const int64_t* slot, const int32_t* used, const void* xbuf,
                                 const void* ybuf, const void* w1, const void* b1, const void* w2, int64_t T,
                                 int32_t k, int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout,
                                 int use_residual, float aux_coef, int normalize_by_k, const int32_t* counts,
                                 void* dx, float* dw1, float* db1, float* dw2, float* db2, float* dlogits,
                                 float* dgate, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(dtype == MOE_F32, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(dy && logits && selected && gates && slot && used && dx && dw1 && db1 && dw2 && db2 && dlogits &&
                    dgate,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(C == 0 || (xbuf && ybuf && w1 && b1 && w2), MOE_ERR_INVALID_ARG);  // unread when C == 0
    MOE_REQUIRE(T >= 1 && k >= 1 && k <= E && E >= 1 && C >= 0 && D >= 1 && F >= 1 && Dout >= 1,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(k <= 64 && E <= 65535, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(!use_residual || Dout == D, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aux_coef == 0.f || counts != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(workspace && workspace_bytes >= moe_backward_gelu_workspace_size(E, C, D, F, Dout),
                MOE_ERR_WORKSPACE);

    const unsigned grid = (unsigned)((T + kWarps - 1) / kWarps);
    launch_dgate<float>(grid, stream, static_cast<const float*>(dy), Dout, static_cast<const float*>(ybuf), logits,
                        selected, gates, slot, T, k, E, C, aux_coef, normalize_by_k ? (float)k : 1.0f, counts, dlogits,
                        dgate, dev_status);
    int rc = launch_status();
    if (rc != MOE_OK) return rc;

    if (C == 0) {  // nothing kept: no expert gradient
        MOE_CUDA_TRY(cudaMemsetAsync(dw1, 0, (size_t)E * F * D * 4, stream));
        MOE_CUDA_TRY(cudaMemsetAsync(db1, 0, (size_t)E * F * 4, stream));
        MOE_CUDA_TRY(cudaMemsetAsync(dw2, 0, (size_t)E * Dout * F * 4, stream));
        MOE_CUDA_TRY(cudaMemsetAsync(db2, 0, (size_t)E * Dout * 4, stream));
        if (use_residual)
            MOE_CUDA_TRY(cudaMemcpyAsync(dx, dy, (size_t)T * D * 4, cudaMemcpyDeviceToDevice, stream));
        else
            MOE_CUDA_TRY(cudaMemsetAsync(dx, 0, (size_t)T * D * 4, stream));
        return MOE_OK;
    }

    const GeluBwdWs l = gelu_bwd_layout(E, C, D, F, Dout);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* dybuf = reinterpret_cast<float*>(ws + l.dybuf);
    float* z = reinterpret_cast<float*>(ws + l.z);
    float* dh = reinterpret_cast<float*>(ws + l.dh);
    float* dxbuf = reinterpret_cast<float*>(ws + l.dxbuf);
    void* split = ws + l.split;
    const size_t split_bytes = workspace_bytes - l.split;
    const float* xb = static_cast<const float*>(xbuf);
    F32Gemm s[5];
    gelu_bwd_shapes(E, C, D, F, Dout, s);
    for (auto& q : s) q.rows = used;
    auto run = [&](const F32Gemm& q) { return tf32x3_gemm_run(q, split, split_bytes, dev_status, stream); };

    // 2. dybuf[e,c] = gate * dy[token]
    rc = gather_rows(dy, Dout, T, k, selected, slot, E, C, gates, dybuf, Dout, MOE_F32, dev_status, stream);
    if (rc != MOE_OK) return rc;
    // 3. z = xbuf W1^T + b1
    s[0].A = xb;
    s[0].B = static_cast<const float*>(w1);
    s[0].bias = static_cast<const float*>(b1);
    s[0].C = z;
    if ((rc = run(s[0])) != MOE_OK) return rc;
    // 4. dh = dybuf W2
    s[1].A = dybuf;
    s[1].B = static_cast<const float*>(w2);
    s[1].C = dh;
    if ((rc = run(s[1])) != MOE_OK) return rc;
    // 5. h = gelu(z) (into z), dz = dh * gelu'(z) (into dh)
    {
        const int64_t blocks = (C * F + 255) / 256;
        const dim3 g2((unsigned)(blocks < 1024 ? blocks : 1024), (unsigned)E);
        gelu_bwd_elem_kernel<<<g2, 256, 0, stream>>>(z, dh, used, C, F);
        if ((rc = launch_status()) != MOE_OK) return rc;
    }
    // 6. dW2 = dybuf^T h,  dW1 = dz^T xbuf
    s[2].A = dybuf;
    s[2].B = z;
    s[2].C = dw2;
    if ((rc = run(s[2])) != MOE_OK) return rc;
    s[3].A = dh;
    s[3].B = xb;
    s[3].C = dw1;
    if ((rc = run(s[3])) != MOE_OK) return rc;
    // 7. bias gradients
    group_column_sum_kernel<<<dim3((unsigned)((Dout + 255) / 256), (unsigned)E), 256, 0, stream>>>(dybuf, C, Dout,
                                                                                                   used, db2);
    if ((rc = launch_status()) != MOE_OK) return rc;
    group_column_sum_kernel<<<dim3((unsigned)((F + 255) / 256), (unsigned)E), 256, 0, stream>>>(dh, C, F, used, db1);
    if ((rc = launch_status()) != MOE_OK) return rc;
    // 8. dxbuf = dz W1
    s[4].A = dh;
    s[4].B = static_cast<const float*>(w1);
    s[4].C = dxbuf;
    if ((rc = run(s[4])) != MOE_OK) return rc;
    // 9. dx
    return combine_rows(dxbuf, selected, slot, nullptr, MOE_F32, T, k, E, C, D, use_residual ? dy : nullptr, D, dx, D,
                        MOE_F32, dev_status, stream);
}
