// moe_expert_ffn: the expert FFNs as grouped GEMMs over variable-occupancy
// experts, on the tcgen05 tensor cores: bf16 operands directly (tc_gemm,
// tcx), fp32 operands as split-tf32 products (tc_tf32).
#include <cuda_runtime.h>

#include "common.cuh"
#include "f32_gemm.cuh"
#include "tc_expert_gemm.cuh"
#include "tc_gemm.cuh"
#include "tc_tf32.cuh"

using namespace moe;

namespace {

// The fp32 GEMMs of one moe_expert_ffn call in F32Gemm form (operand
// pointers left empty): [0] the first projection (LINEAR: the only one),
// [1] the second projection of the MLP experts.
void fp32_shapes(moe_ffn_kind kind, int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout, F32Gemm (&s)[2]) {
    s[0] = F32Gemm{};
    s[0].M = C;
    s[0].K = D;
    s[0].N = kind == MOE_FFN_LINEAR ? Dout : F;
    s[0].groups = E;
    s[1] = F32Gemm{};
    s[1].M = C;
    s[1].K = F;
    s[1].N = Dout;
    s[1].groups = E;
}

size_t fp32_split_bytes(moe_ffn_kind kind, int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout) {
    F32Gemm s[2];
    fp32_shapes(kind, E, C, D, F, Dout, s);
    size_t b = tf32x3_workspace_size(s[0]);
    if (kind != MOE_FFN_LINEAR) {
        const size_t b2 = tf32x3_workspace_size(s[1]);
        b = b2 > b ? b2 : b;
    }
    return b;
}

}  // namespace

namespace {
constexpr size_t kTileCounterBytes = 256;  // after the intermediate h: scratch words of the wide GEMM's scheduler
}

extern "C" size_t moe_expert_ffn_workspace_size(moe_ffn_kind kind, moe_dtype dtype, int32_t E, int64_t C, int64_t D,
                                                int64_t F, int64_t Dout) {
    if (E < 1 || C < 1) return 0;
    size_t h = 0;
    if (kind != MOE_FFN_LINEAR && F >= 1) h = align_up((size_t)E * C * F * dtype_size(dtype), 1024);
    if (dtype == MOE_F32 && D >= 1 && Dout >= 1 && (kind == MOE_FFN_LINEAR || F >= 1))
        return h + fp32_split_bytes(kind, E, C, D, F, Dout);
    if (kind == MOE_FFN_SWIGLU && F >= 1) h += kTileCounterBytes;  // the wide GEMM's tile counter
    return h;
}

namespace {

// Second GEMM of the bf16 MLP experts: ybuf = h (E*C, F) x W2^T (+ b2).
int down_projection(moe_ffn_kind kind, const void* h, const int32_t* used, int32_t E, int64_t C, int64_t F,
                    int64_t Dout, const void* w2, const void* b2, void* ybuf, int32_t* dev_status,
                    cudaStream_t stream) {
    TcGemmProblem q{};
    q.a = h;
    q.lda = F;
    q.a_rows_total = (int64_t)E * C;
    q.a_rows_per_group = C;
    q.b = w2;
    q.ldb = F;
    q.b_rows_total = (int64_t)E * Dout;
    q.b_rows_per_group = Dout;
    q.G = E;
    q.M = C;
    q.N = Dout;
    q.K = F;
    q.rows = used;
    q.out = ybuf;
    q.ldo = Dout;
    q.out_rows_per_group = C;
    q.status = dev_status;
    if (kind == MOE_FFN_GELU_MLP) {
        q.bias = b2;
        q.bias_group_stride = Dout;
        q.epilogue = TC_EPI_BF16_BIAS;
    } else {
        q.epilogue = TC_EPI_BF16;
    }
    return tc_gemm_run(q, stream);
}

}  // namespace

namespace moe {
namespace {
int expert_ffn(moe_ffn_kind kind, moe_dtype dtype, const void* xbuf, const int32_t* used, int32_t E, int64_t C,
               int64_t D, int64_t F, int64_t Dout, const void* w1, const void* b1, const void* w2, const void* b2,
               const void* w3, void* ybuf, void* saved_ab, int32_t* dev_status, void* workspace,
               size_t workspace_bytes, cudaStream_t stream);
}  // namespace
}  // namespace moe

extern "C" int moe_expert_ffn(moe_ffn_kind kind, moe_dtype dtype, const void* xbuf, const int32_t* used, int32_t E,
                              int64_t C, int64_t D, int64_t F, int64_t Dout, const void* w1, const void* b1,
                              const void* w2, const void* b2, const void* w3, void* ybuf, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    return expert_ffn(kind, dtype, xbuf, used, E, C, D, F, Dout, w1, b1, w2, b2, w3, ybuf, nullptr, dev_status,
                      workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int moe_expert_ffn_save(const void* xbuf, const int32_t* used, int32_t E, int64_t C, int64_t D, int64_t F,
                                   int64_t Dout, const void* w_gate, const void* w_down, const void* w_up,
                                   void* ybuf, void* saved_ab, int32_t* dev_status, void* workspace,
                                   size_t workspace_bytes, moe_stream_t stream) {
    MOE_REQUIRE(C == 0 || (used != nullptr && saved_ab != nullptr), MOE_ERR_INVALID_ARG);
    return expert_ffn(MOE_FFN_SWIGLU, MOE_BF16, xbuf, used, E, C, D, F, Dout, w_gate, nullptr, w_down, nullptr, w_up,
                      ybuf, saved_ab, dev_status, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

namespace moe {
namespace {
int expert_ffn(moe_ffn_kind kind, moe_dtype dtype, const void* xbuf, const int32_t* used, int32_t E, int64_t C,
               int64_t D, int64_t F, int64_t Dout, const void* w1, const void* b1, const void* w2, const void* b2,
               const void* w3, void* ybuf, void* saved_ab, int32_t* dev_status, void* workspace,
               size_t workspace_bytes, cudaStream_t stream) {
    MOE_REQUIRE(valid_dtype(dtype), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(kind == MOE_FFN_LINEAR || kind == MOE_FFN_GELU_MLP || kind == MOE_FFN_SWIGLU, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(E >= 1 && C >= 0 && D >= 1 && Dout >= 1, MOE_ERR_INVALID_ARG);
    if (C == 0) return MOE_OK;  // no rows: nothing is read or written
    MOE_REQUIRE(xbuf && ybuf && w1, MOE_ERR_INVALID_ARG);
    if (kind == MOE_FFN_GELU_MLP) MOE_REQUIRE(b1 && w2 && b2 && F >= 1, MOE_ERR_INVALID_ARG);
    if (kind == MOE_FFN_SWIGLU) MOE_REQUIRE(w2 && w3 && F >= 1, MOE_ERR_INVALID_ARG);
    void* h = nullptr;
    const size_t need = moe_expert_ffn_workspace_size(kind, dtype, E, C, D, F, Dout);
    MOE_REQUIRE(need == 0 || (workspace && workspace_bytes >= need), MOE_ERR_WORKSPACE);
    size_t h_bytes = 0;
    if (kind != MOE_FFN_LINEAR) {
        h = workspace;
        h_bytes = align_up((size_t)E * C * F * dtype_size(dtype), 1024);
    }

    if (dtype == MOE_BF16) {
        // Kernel choice (measured on B200): the SwiGLU gate/up GEMM over ragged
        // experts runs with weights on the MMA's M side and up to 256 tokens on N
        // (tcw_gemm_run: at most 15 padded token rows per expert, and the fewest
        // operand bytes per FLOP through the TMA); every other bf16 GEMM runs with
        // token rows on the M side and a single N=256 weight operand (tc_gemm_run).
        int rc;
        if (kind == MOE_FFN_SWIGLU && used != nullptr) {
            TcxProblem p{};
            p.w = w1;   // gate
            p.w2 = w3;  // up
            p.ldw = D;
            p.w_rows_total = (int64_t)E * F;
            p.w_rows_per_group = F;
            p.x = xbuf;
            p.ldx = D;
            p.x_rows_total = (int64_t)E * C;
            p.x_rows_per_group = C;
            p.G = E;
            p.features = F;
            p.max_tokens = C;
            p.K = D;
            p.rows = used;
            p.out = h;
            p.ldo = F;
            p.out_rows_per_group = C;
            p.epilogue = TC_EPI_SWIGLU;
            p.status = dev_status;
            p.save_ab = saved_ab;
            p.ld_save = 2 * F;
            p.tile_counter = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + h_bytes);
            rc = tcw_gemm_run(p, stream);
        } else {
            // first GEMM: xbuf (E*C, D) x W^T
            TcGemmProblem p{};
            p.a = xbuf;
            p.lda = D;
            p.a_rows_total = (int64_t)E * C;
            p.a_rows_per_group = C;
            p.G = E;
            p.M = C;
            p.K = D;
            p.rows = used;
            p.out_rows_per_group = C;
            p.status = dev_status;
            if (kind == MOE_FFN_LINEAR) {
                p.b = w1;
                p.ldb = D;
                p.b_rows_total = (int64_t)E * Dout;
                p.b_rows_per_group = Dout;
                p.N = Dout;
                p.out = ybuf;
                p.ldo = Dout;
                p.epilogue = TC_EPI_BF16;
                return tc_gemm_run(p, stream);
            }
            p.ldb = D;
            p.b_rows_total = (int64_t)E * F;
            p.b_rows_per_group = F;
            p.N = F;
            p.out = h;
            p.ldo = F;
            if (kind == MOE_FFN_SWIGLU) {
                p.b = w1;   // gate
                p.b2 = w3;  // up
                p.epilogue = TC_EPI_SWIGLU;
            } else {
                p.b = w1;
                p.bias = b1;
                p.bias_group_stride = F;
                p.epilogue = TC_EPI_GELU_BIAS;
            }
            rc = tc_gemm_run(p, stream);
        }
        if (rc != MOE_OK) return rc;
        return down_projection(kind, h, used, E, C, F, Dout, w2, b2, ybuf, dev_status, stream);
    }

    // fp32: split-tf32 tensor-core GEMMs, B = weights in (out, in) layout -> transposed operand
    void* split = static_cast<uint8_t*>(workspace) + h_bytes;
    const size_t split_bytes = workspace_bytes - h_bytes;
    auto run = [&](const F32Gemm& q) { return tf32x3_gemm_run(q, split, split_bytes, dev_status, stream); };
    F32Gemm g{};
    g.A = static_cast<const float*>(xbuf);
    g.lda = D;
    g.a_group_stride = C * D;
    g.b_trans = true;
    g.M = C;
    g.K = D;
    g.groups = E;
    g.rows = used;
    g.rows_mode = used ? 1 : 0;
    if (kind == MOE_FFN_LINEAR) {
        g.B = static_cast<const float*>(w1);
        g.ldb = D;
        g.b_group_stride = Dout * D;
        g.C = static_cast<float*>(ybuf);
        g.ldc = Dout;
        g.c_group_stride = C * Dout;
        g.N = Dout;
        return run(g);
    }
    float* hf = static_cast<float*>(h);
    g.ldb = D;
    g.b_group_stride = F * D;
    g.C = hf;
    g.ldc = F;
    g.c_group_stride = C * F;
    g.N = F;
    int rc;
    if (kind == MOE_FFN_GELU_MLP) {
        g.B = static_cast<const float*>(w1);
        g.bias = static_cast<const float*>(b1);
        g.bias_group_stride = F;
        g.epilogue = F32_EPI_BIAS_GELU;
        rc = run(g);
    } else {
        g.B = static_cast<const float*>(w3);  // up -> h
        rc = run(g);
        if (rc != MOE_OK) return rc;
        g.B = static_cast<const float*>(w1);  // gate: h = silu(gate) * up
        g.epilogue = F32_EPI_SILU_MUL;
        rc = run(g);
    }
    if (rc != MOE_OK) return rc;
    F32Gemm d{};
    d.A = hf;
    d.lda = F;
    d.a_group_stride = C * F;
    d.B = static_cast<const float*>(w2);
    d.ldb = F;
    d.b_trans = true;
    d.b_group_stride = Dout * F;
    d.C = static_cast<float*>(ybuf);
    d.ldc = Dout;
    d.c_group_stride = C * Dout;
    d.M = C;
    d.N = Dout;
    d.K = F;
    d.groups = E;
    d.rows = used;
    d.rows_mode = used ? 1 : 0;
    if (kind == MOE_FFN_GELU_MLP) {
        d.bias = static_cast<const float*>(b2);
        d.bias_group_stride = Dout;
        d.epilogue = F32_EPI_BIAS;
    }
    return run(d);
}
}  // namespace
}  // namespace moe

extern "C" int moe_expert_ffn_gathered(moe_ffn_kind kind, moe_dtype dtype, const void* x, int64_t T, int64_t ldx,
                                       const int32_t* token_of_slot, const int32_t* used, int32_t E, int64_t C,
                                       int64_t D, int64_t F, int64_t Dout, const void* w1, const void* w2,
                                       const void* w3, void* ybuf, int32_t* dev_status, void* workspace,
                                       size_t workspace_bytes, moe_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    MOE_REQUIRE(kind == MOE_FFN_SWIGLU && dtype == MOE_BF16, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(T >= 1 && ldx >= D && E >= 1 && C >= 0 && D >= 1 && F >= 1 && Dout >= 1, MOE_ERR_INVALID_ARG);
    if (C == 0) return MOE_OK;  // no rows: nothing is read or written
    MOE_REQUIRE(x && token_of_slot && used && ybuf && w1 && w2 && w3, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(workspace && workspace_bytes >= moe_expert_ffn_workspace_size(kind, dtype, E, C, D, F, Dout),
                MOE_ERR_WORKSPACE);
    void* h = workspace;
    // gate/up with the token rows read from x through token_of_slot
    TcxProblem p{};
    p.w = w1;   // gate
    p.w2 = w3;  // up
    p.ldw = D;
    p.w_rows_total = (int64_t)E * F;
    p.w_rows_per_group = F;
    p.x = x;
    p.ldx = ldx;
    p.x_rows_total = T;
    p.x_rows_per_group = 0;
    p.G = E;
    p.features = F;
    p.max_tokens = C;
    p.K = D;
    p.rows = used;
    p.gather_index = token_of_slot;
    p.out = h;
    p.ldo = F;
    p.out_rows_per_group = C;
    p.epilogue = TC_EPI_SWIGLU;
    p.status = dev_status;
    const int rc = tcx_gemm_run(p, stream);
    if (rc != MOE_OK) return rc;
    return down_projection(kind, h, used, E, C, F, Dout, w2, nullptr, ybuf, dev_status, stream);
}
