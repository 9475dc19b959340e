"""Whole-layer forward passes built from the C-ABI calls, buffers allocated once.

Each ``forward`` enqueues the layer's kernels on the current stream in the order
route -> dispatch -> expert FFN -> combine -> load statistics and returns device
tensors; nothing is synchronised.
"""
from __future__ import annotations

import torch

from . import binding as B


class SwiGLUMoE:
    """Router GEMM + SwiGLU routed experts + optional always-on shared SwiGLU expert.

    y = shared(x) + sum_{kept j} gate_j * Expert_{e_j}(x)   (or no shared term)
    """

    def __init__(self, T: int, H: int, E: int, F: int, k: int, capacity_factor: float, F_shared: int = 0,
                 aux_coef: float = 0.0, dtype=torch.bfloat16, device="cuda", gathered: bool = False,
                 save_for_backward: bool = False):
        self.T, self.H, self.E, self.F, self.k = T, H, E, F, k
        self.F_shared, self.aux_coef, self.dtype = F_shared, aux_coef, dtype
        self.C = B.moe_capacity(T, k, E, capacity_factor)
        dev = torch.device(device)
        dt = B.MOE_BF16 if dtype == torch.bfloat16 else B.MOE_F32
        C = self.C
        self.route_out = dict(
            selected=torch.empty(T, k, dtype=torch.int64, device=dev),
            gates=torch.empty(T, k, dtype=dtype, device=dev),
            gates_f32=torch.empty(T, k, dtype=torch.float32, device=dev),
            counts=torch.empty(E, dtype=torch.int32, device=dev),
            prob_sum=torch.empty(E, dtype=torch.float32, device=dev),
        )
        self.disp_out = dict(
            slot=torch.empty(T, k, dtype=torch.int64, device=dev),
            kept=torch.empty(T, k, dtype=torch.uint8, device=dev),
            used=torch.empty(E, dtype=torch.int32, device=dev),
            overflow=torch.empty(E, dtype=torch.int32, device=dev),
            drops=torch.empty(T, dtype=torch.int32, device=dev),
            token_of_slot=torch.empty(E, C, dtype=torch.int32, device=dev),
        )
        # gathered=True (bf16 only) skips the (E, C, H) copy of the token rows: the
        # expert kernel reads them from x, which saves that memory at about the
        # same step time; otherwise the dispatch gathers them into xbuf.
        self.gathered = gathered and dtype == torch.bfloat16
        if not self.gathered:
            self.disp_out["xbuf"] = torch.empty(E, C, H, dtype=dtype, device=dev)
        self.ybuf = torch.empty(E, C, H, dtype=dtype, device=dev)
        # save_for_backward (bf16, not gathered): the routed experts also keep their gate/up
        # pre-activations (E, C, 2F) for moe_backward_swiglu, which then skips recomputing them
        self.saved_ab = (torch.empty(E, C, 2 * F, dtype=dtype, device=dev)
                         if save_for_backward and dtype == torch.bfloat16 and not self.gathered else None)
        self.y = torch.empty(T, H, dtype=dtype, device=dev)
        self.shared = torch.empty(T, H, dtype=dtype, device=dev) if F_shared else None
        self.status = B.new_status(dev)
        self.ws_route = torch.empty(max(B.moe_route_workspace_size(T, H, E, dt, True, "ED"), 256),
                                    dtype=torch.uint8, device=dev)
        self.ws_disp = torch.empty(max(B.moe_dispatch_workspace_size(T, k, E), 256), dtype=torch.uint8, device=dev)
        self.ws_ffn = torch.empty(max(B.moe_expert_ffn_workspace_size("swiglu", dt, E, C, H, F, H), 256),
                                  dtype=torch.uint8, device=dev)
        self.ws_shared = (torch.empty(max(B.moe_expert_ffn_workspace_size("swiglu", dt, 1, T, H, F_shared, H), 256),
                                      dtype=torch.uint8, device=dev) if F_shared else None)
        self.side = None  # stream for the shared expert, created on first use

    def forward(self, x, w_router, router_bias, w_gate, w_up, w_down, s_gate=None, s_up=None, s_down=None):
        """x (T,H); w_router (E,H); w_gate/w_up (E,F,H); w_down (E,H,F); shared (1,F_s,H)/(1,H,F_s).

        The shared expert only needs x, so it runs on a second stream while the
        router, the slot scan and the gather (short, latency- and memory-bound
        kernels) run on the current one; the combine waits for both.
        """
        main = torch.cuda.current_stream(x.device)
        base_kind, base = "zero", None
        if self.F_shared:
            if self.side is None:
                self.side = torch.cuda.Stream(device=x.device)
                self.ev_x, self.ev_shared = torch.cuda.Event(), torch.cuda.Event()
            self.ev_x.record(main)
            self.side.wait_event(self.ev_x)
            B.moe_expert_ffn("swiglu", x.view(1, self.T, self.H), None, s_gate, w2=s_down, w3=s_up,
                             ybuf=self.shared.view(1, self.T, self.H), dev_status=self.status,
                             workspace=self.ws_shared, stream=self.side)
            self.ev_shared.record(self.side)
            base_kind, base = "tensor", self.shared
        r = B.moe_route(x, self.k, w_router=w_router, layout="ED", logit_bias=router_bias, out=self.route_out,
                        dev_status=self.status, workspace=self.ws_route)
        if self.gathered:  # slots only: the expert kernel reads its rows from x through token_of_slot
            d = B.moe_dispatch(r["selected"], self.E, self.C, out=self.disp_out, dev_status=self.status,
                               workspace=self.ws_disp)
            B.moe_expert_ffn_gathered(x, d["token_of_slot"], d["used"], w_gate, w_down, w_up, ybuf=self.ybuf,
                                      dev_status=self.status, workspace=self.ws_ffn)
        else:
            d = B.moe_dispatch(r["selected"], self.E, self.C, x=x, out=self.disp_out, dev_status=self.status,
                               workspace=self.ws_disp)
            if self.saved_ab is not None:
                B.moe_expert_ffn_save(d["xbuf"], d["used"], w_gate, w_down, w_up, self.saved_ab, ybuf=self.ybuf,
                                      dev_status=self.status, workspace=self.ws_ffn)
            else:
                B.moe_expert_ffn("swiglu", d["xbuf"], d["used"], w_gate, w2=w_down, w3=w_up, ybuf=self.ybuf,
                                 dev_status=self.status, workspace=self.ws_ffn)
        if self.F_shared:
            main.wait_event(self.ev_shared)
        B.moe_combine(self.ybuf, r["selected"], d["slot"], r["gates_f32"], base_kind=base_kind, base=base, y=self.y,
                      dev_status=self.status)
        f, P, aux = B.moe_aux_stats(r["counts"], r["prob_sum"], self.T, self.k, True, self.aux_coef,
                                    out_dtype=self.dtype)
        return dict(y=self.y, f=f, P=P, aux=aux, **r, **d)


class SwiGLULayer:
    """The same layer as SwiGLUMoE through the single C call moe_swiglu_layer_forward.

    Holds the layer description (sizes and device weight pointers) and one
    workspace per in-flight batch; ``forward`` accepts x and y on the device or
    in (pinned) host memory, in which case the library does the copies.
    """

    def __init__(self, T: int, H: int, E: int, F: int, k: int, capacity_factor: float, w_router, router_bias, w_gate,
                 w_up, w_down, s_gate=None, s_up=None, s_down=None, aux_coef: float = 0.0, n_workspaces: int = 1,
                 device="cuda"):
        self.C = B.moe_capacity(T, k, E, capacity_factor)
        F_shared = 0 if s_gate is None else int(s_gate.shape[1])
        self._keep = [w_router, router_bias, w_gate, w_up, w_down, s_gate, s_up, s_down]
        d = B.SwiGLULayerDesc()
        d.T, d.H, d.F, d.F_shared, d.C, d.E, d.k, d.aux_coef = T, H, F, F_shared, self.C, E, k, aux_coef
        for name, t in (("w_router", w_router), ("router_bias", router_bias), ("w_gate", w_gate), ("w_up", w_up),
                        ("w_down", w_down), ("s_gate", s_gate), ("s_up", s_up), ("s_down", s_down)):
            setattr(d, name, None if t is None else t.data_ptr())
        self.desc = d
        nbytes = B.moe_swiglu_layer_workspace_size(d)
        if nbytes == 0:
            raise ValueError("invalid layer description")
        self.workspaces = [torch.empty(nbytes, dtype=torch.uint8, device=device) for _ in range(n_workspaces)]
        self.x_free = [torch.cuda.Event() for _ in range(n_workspaces)]
        self.y_free = [torch.cuda.Event() for _ in range(n_workspaces)]
        self.status = B.new_status(device)

    def forward(self, x, y, aux=None, slot: int = 0, stream=None, side_stream=None, copy_in_stream=None,
                copy_out_stream=None):
        """Enqueue one batch on workspace ``slot``; returns y (complete once the copy-out stream gets there)."""
        return B.moe_swiglu_layer_forward(self.desc, x, y, aux, self.workspaces[slot], dev_status=self.status,
                                          stream=stream, side_stream=side_stream, copy_in_stream=copy_in_stream,
                                          copy_out_stream=copy_out_stream, x_free=self.x_free[slot],
                                          y_free=self.y_free[slot])
