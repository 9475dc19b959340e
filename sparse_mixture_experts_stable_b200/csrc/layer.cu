// moe_swiglu_layer_forward: the whole forward of Module 7's EducationalMoE
// (router, capacity-limited dispatch, SwiGLU routed experts, an optional
// always-on shared SwiGLU expert, gate-weighted combine, load statistics) as
// one call on caller-owned memory.
//
// The activations and the output may live on the host: then the call copies x
// into the workspace (one cudaMemcpyAsync on the copy-in stream) and y and the
// aux loss back (one cudaMemcpyAsync each on the copy-out stream).  With
// separate copy streams and two events per workspace (its x staging free, its y
// staging free), consecutive calls on two workspaces overlap one batch's copy-in,
// the previous batch's copy-out and the kernels in between.
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {
namespace {

struct LayerWs {
    size_t x, y, selected, gates, gates_f32, counts, prob_sum, slot, kept, used, overflow, drops, tos, xbuf, ybuf,
        shared, f, P, aux, ws_route, ws_disp, ws_ffn, ws_shared, total;
    size_t n_route, n_disp, n_ffn, n_shared;
};

LayerWs layer_ws(const moe_swiglu_layer* L) {
    LayerWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align_up(bytes > 0 ? bytes : 1, 256);
        return o;
    };
    const size_t T = (size_t)L->T, H = (size_t)L->H, E = (size_t)L->E, k = (size_t)L->k, C = (size_t)L->C;
    w.x = take(T * H * 2);
    w.y = take(T * H * 2);
    w.selected = take(T * k * 8);
    w.gates = take(T * k * 2);
    w.gates_f32 = take(T * k * 4);
    w.counts = take(E * 4);
    w.prob_sum = take(E * 4);
    w.slot = take(T * k * 8);
    w.kept = take(T * k);
    w.used = take(E * 4);
    w.overflow = take(E * 4);
    w.drops = take(T * 4);
    w.tos = take(E * C * 4);
    w.xbuf = take(E * C * H * 2);
    w.ybuf = take(E * C * H * 2);
    w.shared = take(L->F_shared > 0 ? T * H * 2 : 0);
    w.f = take(E * 2);
    w.P = take(E * 2);
    w.aux = take(2 * 4);
    w.n_route = moe_route_workspace_size(L->T, L->H, L->E, MOE_BF16, 1, MOE_ROUTER_ED);
    w.ws_route = take(w.n_route);
    w.n_disp = moe_dispatch_workspace_size(L->T, L->k, L->E);
    w.ws_disp = take(w.n_disp);
    w.n_ffn = moe_expert_ffn_workspace_size(MOE_FFN_SWIGLU, MOE_BF16, L->E, L->C, L->H, L->F, L->H);
    w.ws_ffn = take(w.n_ffn);
    w.n_shared = L->F_shared > 0
                     ? moe_expert_ffn_workspace_size(MOE_FFN_SWIGLU, MOE_BF16, 1, L->T, L->H, L->F_shared, L->H)
                     : 0;
    w.ws_shared = take(w.n_shared);
    w.total = off;
    return w;
}

int check_layer(const moe_swiglu_layer* L) {
    MOE_REQUIRE(L != nullptr, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(L->T >= 1 && L->H >= 1 && L->F >= 1 && L->F_shared >= 0 && L->C >= 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(L->E >= 1 && L->k >= 1 && L->k <= L->E, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(L->w_router && L->w_gate && L->w_up && L->w_down, MOE_ERR_INVALID_ARG);
    if (L->F_shared > 0) MOE_REQUIRE(L->s_gate && L->s_up && L->s_down, MOE_ERR_INVALID_ARG);
    return MOE_OK;
}

// 1 if p is memory the host addresses directly (pinned or pageable), 0 if device memory.
int is_host_ptr(const void* p, int* host) {
    cudaPointerAttributes a{};
    MOE_CUDA_TRY(cudaPointerGetAttributes(&a, p));
    *host = (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeUnregistered) ? 1 : 0;
    return MOE_OK;
}

// Events that order the streams inside one call; destroyed when the call returns
// (a destroyed event that is still pending is released once it completes).
struct CallEvents {
    cudaEvent_t e[4] = {nullptr, nullptr, nullptr, nullptr};
    int n = 0;
    ~CallEvents() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(e[i]);
    }
    cudaEvent_t make() {
        if (n == 4) return nullptr;
        if (cudaEventCreateWithFlags(&e[n], cudaEventDisableTiming) != cudaSuccess) return nullptr;
        return e[n++];
    }
};

// `waiter` waits for everything enqueued on `on` so far.
int order_after(cudaStream_t waiter, cudaStream_t on, CallEvents& ev) {
    if (waiter == on) return MOE_OK;
    cudaEvent_t e = ev.make();
    MOE_REQUIRE(e != nullptr, MOE_ERR_CUDA);
    MOE_CUDA_TRY(cudaEventRecord(e, on));
    MOE_CUDA_TRY(cudaStreamWaitEvent(waiter, e, 0));
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_swiglu_layer_workspace_size(const moe_swiglu_layer* L) {
    if (check_layer(L) != MOE_OK) return 0;
    return layer_ws(L).total;
}

extern "C" int moe_swiglu_layer_forward(const moe_swiglu_layer* L, const void* x, void* y, float* aux,
                                        int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                        moe_stream_t stream_, moe_stream_t side_stream_, moe_stream_t copy_in_,
                                        moe_stream_t copy_out_, moe_event_t x_free_, moe_event_t y_free_) {
    int rc = check_layer(L);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(x && y, MOE_ERR_INVALID_ARG);
    const LayerWs w = layer_ws(L);
    MOE_REQUIRE(workspace != nullptr && workspace_bytes >= w.total, MOE_ERR_WORKSPACE);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    cudaStream_t side = side_stream_ ? reinterpret_cast<cudaStream_t>(side_stream_) : s;
    cudaStream_t cin = copy_in_ ? reinterpret_cast<cudaStream_t>(copy_in_) : s;
    cudaStream_t cout = copy_out_ ? reinterpret_cast<cudaStream_t>(copy_out_) : s;
    cudaEvent_t x_free = reinterpret_cast<cudaEvent_t>(x_free_);
    cudaEvent_t y_free = reinterpret_cast<cudaEvent_t>(y_free_);
    int x_host = 0, y_host = 0, aux_host = 0;
    if ((rc = is_host_ptr(x, &x_host)) != MOE_OK) return rc;
    if ((rc = is_host_ptr(y, &y_host)) != MOE_OK) return rc;
    if (aux && (rc = is_host_ptr(aux, &aux_host)) != MOE_OK) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
    const int64_t T = L->T, H = L->H, C = L->C;
    const int32_t E = L->E, k = L->k;
    CallEvents ev;

    // The previous call on this workspace: its kernels are done with everything but the y staging
    // once x_free fires, and its copy-out is done once y_free fires.  Activations that live on the
    // host are copied into the workspace.
    if (x_free) MOE_CUDA_TRY(cudaStreamWaitEvent(x_host ? cin : s, x_free, 0));
    const void* xd = x;
    if (x_host) {
        if (!x_free && (rc = order_after(cin, s, ev)) != MOE_OK) return rc;
        MOE_CUDA_TRY(cudaMemcpyAsync(at(w.x), x, (size_t)(T * H * 2), cudaMemcpyHostToDevice, cin));
        if ((rc = order_after(s, cin, ev)) != MOE_OK) return rc;
        xd = at(w.x);
    }

    // the always-on shared expert needs only x: it runs on the side stream meanwhile
    moe_base base_kind = MOE_BASE_ZERO;
    if (L->F_shared > 0) {
        if ((rc = order_after(side, s, ev)) != MOE_OK) return rc;
        rc = moe_expert_ffn(MOE_FFN_SWIGLU, MOE_BF16, xd, nullptr, 1, T, H, L->F_shared, H, L->s_gate, nullptr,
                            L->s_down, nullptr, L->s_up, at(w.shared), dev_status, at(w.ws_shared), w.n_shared,
                            reinterpret_cast<moe_stream_t>(side));
        if (rc != MOE_OK) return rc;
        base_kind = MOE_BASE_TENSOR;
    }
    rc = moe_route(xd, MOE_BF16, T, H, H, L->w_router, MOE_ROUTER_ED, E, L->router_bias, k, nullptr,
                   static_cast<int64_t*>(at(w.selected)), at(w.gates), static_cast<float*>(at(w.gates_f32)),
                   static_cast<int32_t*>(at(w.counts)), static_cast<float*>(at(w.prob_sum)), dev_status,
                   at(w.ws_route), w.n_route, stream_);
    if (rc != MOE_OK) return rc;
    rc = moe_dispatch(static_cast<const int64_t*>(at(w.selected)), T, k, E, C, xd, MOE_BF16, H, H,
                      static_cast<int64_t*>(at(w.slot)), static_cast<uint8_t*>(at(w.kept)),
                      static_cast<int32_t*>(at(w.used)), static_cast<int32_t*>(at(w.overflow)),
                      static_cast<int32_t*>(at(w.drops)), static_cast<int32_t*>(at(w.tos)), at(w.xbuf), dev_status,
                      at(w.ws_disp), w.n_disp, stream_);
    if (rc != MOE_OK) return rc;
    rc = moe_expert_ffn(MOE_FFN_SWIGLU, MOE_BF16, at(w.xbuf), static_cast<const int32_t*>(at(w.used)), E, C, H,
                        L->F, H, L->w_gate, nullptr, L->w_down, nullptr, L->w_up, at(w.ybuf), dev_status,
                        at(w.ws_ffn), w.n_ffn, stream_);
    if (rc != MOE_OK) return rc;
    if (L->F_shared > 0 && (rc = order_after(s, side, ev)) != MOE_OK) return rc;
    if (y_free && (y_host || aux_host)) MOE_CUDA_TRY(cudaStreamWaitEvent(s, y_free, 0));
    void* yd = y_host ? at(w.y) : y;
    rc = moe_combine(at(w.ybuf), static_cast<const int64_t*>(at(w.selected)), static_cast<const int64_t*>(at(w.slot)),
                     at(w.gates_f32), MOE_F32, T, k, E, C, H, base_kind, L->F_shared > 0 ? at(w.shared) : nullptr, H,
                     yd, H, MOE_BF16, dev_status, stream_);
    if (rc != MOE_OK) return rc;
    float* auxd = (aux && !aux_host) ? aux : static_cast<float*>(at(w.aux));
    rc = moe_aux_stats(static_cast<const int32_t*>(at(w.counts)), static_cast<const float*>(at(w.prob_sum)), T, E, k,
                       1, L->aux_coef, at(w.f), at(w.P), MOE_BF16, auxd, stream_);
    if (rc != MOE_OK) return rc;

    // every kernel of this call is enqueued: the next call may refill the x staging after them
    if (x_free) MOE_CUDA_TRY(cudaEventRecord(x_free, s));
    // results back to the host, then the y staging is free for the next call
    if (y_host || aux_host) {
        if ((rc = order_after(cout, s, ev)) != MOE_OK) return rc;
        if (y_host) MOE_CUDA_TRY(cudaMemcpyAsync(y, at(w.y), (size_t)(T * H * 2), cudaMemcpyDeviceToHost, cout));
        if (aux_host) MOE_CUDA_TRY(cudaMemcpyAsync(aux, at(w.aux), 2 * sizeof(float), cudaMemcpyDeviceToHost, cout));
        if (y_free) MOE_CUDA_TRY(cudaEventRecord(y_free, cout));
    }
    return MOE_OK;
}
