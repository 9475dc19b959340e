// Row movement kernels: batched transpose, token-major gather into expert-major
// buffers, and the deterministic gate-weighted combine.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "util_kernels.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

// ------------------------------- transpose ----------------------------------
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t rows, int64_t cols) {
    __shared__ T tile[32][33];
    const int64_t b = blockIdx.z;
    const T* s = src + b * rows * cols;
    T* d = dst + b * rows * cols;
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = s[r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < cols) d[c * rows + r] = tile[threadIdx.x][i];
    }
}

// Per-token assignment table held in two registers per lane (j < 64).
struct Assign {
    int64_t e0, e1, s0, s1;
    float g0, g1;
};

__device__ __forceinline__ void load_assign(Assign& a, int lane, int64_t t, int k, const int64_t* selected,
                                            const int64_t* slot) {
    a.e0 = lane < k ? selected[t * k + lane] : -1;
    a.s0 = lane < k ? slot[t * k + lane] : -1;
    a.e1 = lane + 32 < k ? selected[t * k + lane + 32] : -1;
    a.s1 = lane + 32 < k ? slot[t * k + lane + 32] : -1;
}

__device__ __forceinline__ void get_assign(const Assign& a, int j, int64_t& e, int64_t& s) {
    const int src = j & 31;
    const int64_t e0 = __shfl_sync(0xffffffffu, a.e0, src), e1 = __shfl_sync(0xffffffffu, a.e1, src);
    const int64_t s0 = __shfl_sync(0xffffffffu, a.s0, src), s1 = __shfl_sync(0xffffffffu, a.s1, src);
    e = j < 32 ? e0 : e1;
    s = j < 32 ? s0 : s1;
}

__device__ __forceinline__ float get_gate(const Assign& a, int j) {
    const int src = j & 31;
    const float g0 = __shfl_sync(0xffffffffu, a.g0, src), g1 = __shfl_sync(0xffffffffu, a.g1, src);
    return j < 32 ? g0 : g1;
}

// x <- x * g elementwise for the 16 bytes of x (rounded back to T).
template <typename T>
__device__ __forceinline__ void scale_vec(uint4& x, float g) {
    T* xv = reinterpret_cast<T*>(&x);
#pragma unroll
    for (int i = 0; i < 16 / (int)sizeof(T); ++i) xv[i] = from_f32<T>(to_f32(xv[i]) * g);
}

template <>
__device__ __forceinline__ void scale_vec<float>(uint4& x, float g) {
    x.x = __float_as_uint(__uint_as_float(x.x) * g);
    x.y = __float_as_uint(__uint_as_float(x.y) * g);
    x.z = __float_as_uint(__uint_as_float(x.z) * g);
    x.w = __float_as_uint(__uint_as_float(x.w) * g);
}

// ------------------------------- gather -------------------------------------
// One warp per token; 16-byte vectors when every row start is 16-byte aligned.
// EP: the destination of expert e is rank e / epr's buffer (tab), row
// (e % epr) * C + slot; otherwise dst row e * C + slot.
template <typename T, bool VEC, bool EP>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    gather_kernel(const T* __restrict__ src, int64_t lds, int64_t Ttok, int k, const int64_t* __restrict__ selected,
                  const int64_t* __restrict__ slot, int E, int64_t C, const float* __restrict__ scale,
                  T* __restrict__ dst, int64_t D, int32_t* status, const RankTable tab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
    if (t >= Ttok) return;
    Assign a;
    load_assign(a, lane, t, k, selected, slot);
    a.g0 = (scale && lane < k) ? scale[t * k + lane] : 1.f;
    a.g1 = (scale && lane + 32 < k) ? scale[t * k + lane + 32] : 1.f;
    const T* srow = src + t * lds;
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
    for (int j = 0; j < k; ++j) {
        int64_t e, s;
        get_assign(a, j, e, s);
        if (s < 0) continue;
        if (e < 0 || e >= E || s >= C) {
            if (lane == 0) set_status(status, MOE_ERR_BAD_INDEX);
            continue;
        }
        const float g = get_gate(a, j);
        T* drow = EP ? static_cast<T*>(tab.base[e / tab.epr]) + ((e % tab.epr) * C + s) * D : dst + (e * C + s) * D;
        if (VEC) {
            const int64_t nv = D / EPV;
            for (int64_t v = lane; v < nv; v += 32) {
                uint4 x = reinterpret_cast<const uint4*>(srow)[v];
                if (scale) scale_vec<T>(x, g);
                reinterpret_cast<uint4*>(drow)[v] = x;
            }
        } else {
            for (int64_t d = lane; d < D; d += 32) {
                const float v = to_f32(srow[d]) * (scale ? g : 1.f);
                drow[d] = scale ? from_f32<T>(v) : srow[d];
            }
        }
    }
    if (EP) __threadfence_system();  // rows written to peer memory are visible before the kernel ends
}

// ------------------------------- combine ------------------------------------
// One warp per token.  The token's (row offset, gate) table for j < k is staged
// in shared memory first, so the row loops below contain no warp shuffles and
// may diverge freely over ragged row lengths.
constexpr int kMaxKCombine = 64;
constexpr int kCombineBatch = 4;  // row loads issued before the first add (4 measured faster than 8)

// EP: the row of expert e is read from rank e / epr's buffer (tab), and the
// staged table holds its address instead of an offset into ybuf.
template <typename T, typename G, bool VEC, bool EP>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    combine_kernel(const T* __restrict__ ybuf, const int64_t* __restrict__ selected, const int64_t* __restrict__ slot,
                   const G* __restrict__ gates, int64_t Ttok, int k, int E, int64_t C, int64_t N,
                   const T* __restrict__ base, int64_t ldbase, T* __restrict__ y, int64_t ldy, int32_t* status,
                   const RankTable tab) {
    __shared__ int64_t s_row[kWarpsPerBlock][kMaxKCombine];
    __shared__ float s_gate[kWarpsPerBlock][kMaxKCombine];
    __shared__ int s_n[kWarpsPerBlock];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarpsPerBlock + warp;
    if (t >= Ttok) return;
    // compact the kept, in-range assignments in ascending j: lanes read 32
    // assignments at a time and a ballot gives each kept one its position
    int nk = 0;
    for (int j0 = 0; j0 < k; j0 += 32) {
        const int j = j0 + lane;
        bool keep = false;
        int64_t row = 0;
        float g = 1.f;
        if (j < k) {
            const int64_t s = slot[t * k + j];
            if (s >= 0) {
                const int64_t e = selected[t * k + j];
                if (e < 0 || e >= E || s >= C) {
                    set_status(status, MOE_ERR_BAD_INDEX);
                } else {
                    keep = true;
                    if (EP)
                        row = reinterpret_cast<int64_t>(static_cast<const T*>(tab.base[e / tab.epr]) +
                                                        ((e % tab.epr) * C + s) * N);
                    else
                        row = (e * C + s) * N;
                    if (gates) g = to_f32(gates[t * k + j]);
                }
            }
        }
        const uint32_t m = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const int pos = nk + __popc(m & lanemask_lt());
            s_row[warp][pos] = row;
            s_gate[warp][pos] = g;
        }
        nk += __popc(m);
    }
    if (lane == 0) s_n[warp] = nk;
    __syncwarp();
    const int n_terms = s_n[warp];
    const int64_t* rows = s_row[warp];
    const float* gs = s_gate[warp];
    T* yrow = y + t * ldy;
    const T* brow = base ? base + t * ldbase : nullptr;
    if (VEC) {
        constexpr int EPV = 16 / sizeof(T);
        const int64_t nv = N / EPV;
        for (int64_t v = lane; v < nv; v += 32) {
            float acc[EPV];
            if (brow) {
                const uint4 b = reinterpret_cast<const uint4*>(brow)[v];
                const T* bv = reinterpret_cast<const T*>(&b);
#pragma unroll
                for (int i = 0; i < EPV; ++i) acc[i] = to_f32(bv[i]);
            } else {
#pragma unroll
                for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
            }
            // up to kCombineBatch rows in flight per lane, added in ascending j
            for (int j0 = 0; j0 < n_terms; j0 += kCombineBatch) {
                uint4 r[kCombineBatch];
#pragma unroll
                for (int u = 0; u < kCombineBatch; ++u)
                    if (j0 + u < n_terms) {
                        const T* rp = EP ? reinterpret_cast<const T*>(rows[j0 + u]) : ybuf + rows[j0 + u];
                        r[u] = reinterpret_cast<const uint4*>(rp)[v];
                    }
#pragma unroll
                for (int u = 0; u < kCombineBatch; ++u) {
                    if (j0 + u < n_terms) {
                        const float g = gs[j0 + u];
                        const T* rv = reinterpret_cast<const T*>(&r[u]);
#pragma unroll
                        for (int i = 0; i < EPV; ++i) acc[i] = fmaf(g, to_f32(rv[i]), acc[i]);
                    }
                }
            }
            uint4 o;
            T* ov = reinterpret_cast<T*>(&o);
#pragma unroll
            for (int i = 0; i < EPV; ++i) ov[i] = from_f32<T>(acc[i]);
            reinterpret_cast<uint4*>(yrow)[v] = o;
        }
    } else {
        for (int64_t n = lane; n < N; n += 32) {
            float acc = brow ? to_f32(brow[n]) : 0.f;
            for (int j = 0; j < n_terms; ++j) {
                const T* rp = EP ? reinterpret_cast<const T*>(rows[j]) : ybuf + rows[j];
                acc = fmaf(gs[j], to_f32(rp[n]), acc);
            }
            yrow[n] = from_f32<T>(acc);
        }
    }
}

}  // namespace

int transpose_matrices(const void* src, void* dst, int64_t batches, int64_t rows, int64_t cols, moe_dtype dtype,
                       cudaStream_t stream) {
    MOE_REQUIRE(src && dst && batches >= 1 && rows >= 1 && cols >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(batches <= 65535 && (rows + 31) / 32 <= 65535, MOE_ERR_UNSUPPORTED);
    dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32), (unsigned)batches);
    dim3 block(32, 8);
    if (dtype == MOE_BF16)
        transpose_kernel<uint16_t><<<grid, block, 0, stream>>>(static_cast<const uint16_t*>(src),
                                                               static_cast<uint16_t*>(dst), rows, cols);
    else
        transpose_kernel<float><<<grid, block, 0, stream>>>(static_cast<const float*>(src), static_cast<float*>(dst),
                                                            rows, cols);
    return launch_status();
}

bool RankTable::aligned16_all() const {
    for (int r = 0; r < ranks; ++r)
        if (!aligned16(base[r])) return false;
    return true;
}

template <typename T>
static void launch_gather(bool vec, const RankTable* tab, unsigned grid, const void* src, int64_t lds, int64_t T_,
                          int k, const int64_t* selected, const int64_t* slot, int E, int64_t C, const float* scale,
                          void* dst, int64_t D, int32_t* status, cudaStream_t stream) {
    const int threads = kWarpsPerBlock * 32;
    auto s = static_cast<const T*>(src);
    auto d = static_cast<T*>(dst);
    const RankTable t = tab ? *tab : RankTable{};
    if (tab) {
        if (vec) gather_kernel<T, true, true><<<grid, threads, 0, stream>>>(s, lds, T_, k, selected, slot, E, C, scale, d, D, status, t);
        else gather_kernel<T, false, true><<<grid, threads, 0, stream>>>(s, lds, T_, k, selected, slot, E, C, scale, d, D, status, t);
    } else {
        if (vec) gather_kernel<T, true, false><<<grid, threads, 0, stream>>>(s, lds, T_, k, selected, slot, E, C, scale, d, D, status, t);
        else gather_kernel<T, false, false><<<grid, threads, 0, stream>>>(s, lds, T_, k, selected, slot, E, C, scale, d, D, status, t);
    }
}

int gather_rows(const void* src, int64_t lds, int64_t T, int32_t k, const int64_t* selected, const int64_t* slot,
                int32_t E, int64_t C, const float* scale, void* dst, int64_t D, moe_dtype dtype, int32_t* status,
                cudaStream_t stream, const RankTable* tab) {
    MOE_REQUIRE(k >= 1 && k <= 64, MOE_ERR_UNSUPPORTED);
    if (T == 0 || C == 0 || D == 0) return MOE_OK;
    const size_t es = dtype_size(dtype);
    const bool dst_ok = tab ? tab->aligned16_all() : aligned16(dst);
    const bool vec = aligned16(src) && dst_ok && ((size_t)lds * es) % 16 == 0 && ((size_t)D * es) % 16 == 0;
    const unsigned grid = (unsigned)((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
    if (dtype == MOE_BF16)
        launch_gather<__nv_bfloat16>(vec, tab, grid, src, lds, T, k, selected, slot, E, C, scale, dst, D, status,
                                     stream);
    else
        launch_gather<float>(vec, tab, grid, src, lds, T, k, selected, slot, E, C, scale, dst, D, status, stream);
    return launch_status();
}

template <typename T, typename G, bool EP>
static void launch_combine_ep(bool vec, unsigned grid, const void* ybuf, const int64_t* selected, const int64_t* slot,
                              const void* gates, int64_t T_, int k, int E, int64_t C, int64_t N, const void* base,
                              int64_t ldbase, void* y, int64_t ldy, int32_t* status, const RankTable& tab,
                              cudaStream_t stream) {
    const int threads = kWarpsPerBlock * 32;
    if (vec)
        combine_kernel<T, G, true, EP><<<grid, threads, 0, stream>>>(
            static_cast<const T*>(ybuf), selected, slot, static_cast<const G*>(gates), T_, k, E, C, N,
            static_cast<const T*>(base), ldbase, static_cast<T*>(y), ldy, status, tab);
    else
        combine_kernel<T, G, false, EP><<<grid, threads, 0, stream>>>(
            static_cast<const T*>(ybuf), selected, slot, static_cast<const G*>(gates), T_, k, E, C, N,
            static_cast<const T*>(base), ldbase, static_cast<T*>(y), ldy, status, tab);
}

template <typename T, typename G>
static void launch_combine(bool vec, unsigned grid, const void* ybuf, const int64_t* selected, const int64_t* slot,
                           const void* gates, int64_t T_, int k, int E, int64_t C, int64_t N, const void* base,
                           int64_t ldbase, void* y, int64_t ldy, int32_t* status, const RankTable* tab,
                           cudaStream_t stream) {
    if (tab)
        launch_combine_ep<T, G, true>(vec, grid, ybuf, selected, slot, gates, T_, k, E, C, N, base, ldbase, y, ldy,
                                      status, *tab, stream);
    else
        launch_combine_ep<T, G, false>(vec, grid, ybuf, selected, slot, gates, T_, k, E, C, N, base, ldbase, y, ldy,
                                       status, RankTable{}, stream);
}

int combine_rows(const void* ybuf, const int64_t* selected, const int64_t* slot, const void* gates,
                 moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C, int64_t N, const void* base,
                 int64_t ldbase, void* y, int64_t ldy, moe_dtype dtype, int32_t* status, cudaStream_t stream,
                 const RankTable* tab) {
    MOE_REQUIRE(k >= 1 && k <= kMaxKCombine, MOE_ERR_UNSUPPORTED);
    if (T == 0 || N == 0) return MOE_OK;
    const size_t es = dtype_size(dtype);
    const bool src_ok = tab ? tab->aligned16_all() : aligned16(ybuf);
    const bool vec = src_ok && aligned16(y) && (!base || aligned16(base)) && ((size_t)N * es) % 16 == 0 &&
                     ((size_t)ldy * es) % 16 == 0 && (!base || ((size_t)ldbase * es) % 16 == 0);
    const unsigned grid = (unsigned)((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
    if (dtype == MOE_BF16) {
        if (gate_dtype == MOE_BF16)
            launch_combine<__nv_bfloat16, __nv_bfloat16>(vec, grid, ybuf, selected, slot, gates, T, k, E, C, N, base,
                                                         ldbase, y, ldy, status, tab, stream);
        else
            launch_combine<__nv_bfloat16, float>(vec, grid, ybuf, selected, slot, gates, T, k, E, C, N, base, ldbase,
                                                 y, ldy, status, tab, stream);
    } else {
        if (gate_dtype == MOE_BF16)
            launch_combine<float, __nv_bfloat16>(vec, grid, ybuf, selected, slot, gates, T, k, E, C, N, base, ldbase,
                                                 y, ldy, status, tab, stream);
        else
            launch_combine<float, float>(vec, grid, ybuf, selected, slot, gates, T, k, E, C, N, base, ldbase, y, ldy,
                                         status, tab, stream);
    }
    return launch_status();
}

}  // namespace moe
