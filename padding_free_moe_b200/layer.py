"""One padding-free MoE layer: device buffers plus the call sequence of the C ABI.

Host plumbing only -- torch allocates the device buffers once, every compute
step is a libpfmoe kernel.  Forward: moe_route -> pft_build -> moe_dispatch ->
moe_expert_ffn -> moe_combine.  Backward: moe_backward.  RBD: rbd_plan.

fused_gather=True (BF16 only) runs the forward as moe_route -> pft_build ->
moe_expert_ffn_gathered (the first expert GEMM reads its rows from x by token id,
so the forward writes no [N, d] copy of x) -> moe_combine, and the backward as
moe_dispatch (the PFT copy of x, needed only by the weight gradients) ->
moe_backward.  Same results bit for bit; it is off by default because the
gathered GEMM is slower on B200 than dispatch plus the TMA-fed GEMM.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib as L


@dataclass
class Shape:
    T: int
    d: int
    E: int
    h: int
    k: int
    dtype: torch.dtype
    rbd_epd: Optional[int] = None
    rbd_dpn: Optional[int] = None

    @property
    def N(self) -> int:
        return self.T * self.k


class PFTMoELayer:
    """Buffers for one layer shape on one device; inputs/weights are passed per call."""

    def __init__(self, shape: Shape, device="cuda", fused_gather=False):
        self.s = s = shape
        self.device = torch.device(device)
        self.code = L.dtype_code(s.dtype)
        self.fused_gather = bool(fused_gather) and s.dtype == torch.bfloat16
        dev, f32, i32, dt = self.device, torch.float32, torch.int32, s.dtype
        T, d, E, h, k, N = s.T, s.d, s.E, s.h, s.k, s.N
        e = lambda *shape_, dtype=dt: torch.empty(*shape_, device=dev, dtype=dtype)
        # routing + PFT
        self.logits = e(T, E, dtype=f32)
        self.topk_ids = e(T, k, dtype=i32)
        self.topk_w = e(T, k, dtype=f32)
        self.route_ws_bytes = L.moe_route_workspace_size(T, d, E, k, self.code)
        self.route_ws = e(max(self.route_ws_bytes, 256), dtype=torch.uint8)
        self.tokens_per_expert = e(E, dtype=i32)
        self.expert_offsets = e(E + 1, dtype=i32)
        self.token_ids = e(max(N, 1), dtype=i32)
        self.expert_ids = e(max(N, 1), dtype=i32)
        self.combine_weights = e(max(N, 1), dtype=f32)
        self.pos = e(T, k, dtype=i32)
        self.tile_offsets = e(E + 1, dtype=i32)
        self.pft_ws_bytes = L.pft_build_workspace_size(T, E, k)
        self.pft_ws = e(max(self.pft_ws_bytes, 256), dtype=torch.uint8)
        # activations
        self.x_pft = e(max(N, 1), d)
        self.h1 = e(max(N, 1), h)
        self.h3 = e(max(N, 1), h)
        self.a = e(max(N, 1), h)
        self.out = e(max(N, 1), d)
        self.y = e(T, d)
        # gradients
        self.dx = e(T, d)
        self.dwg = e(d, E, dtype=f32)
        self.dw1 = e(E, d, h)
        self.dw3 = e(E, d, h)
        self.dw2 = e(E, h, d)
        self.dlogits = e(T, E, dtype=f32)
        self.bwd_ws_bytes = L.moe_backward_workspace_size(T, d, E, h, k, self.code)
        self.bwd_ws = e(max(self.bwd_ws_bytes, 256), dtype=torch.uint8)
        self.err = torch.zeros(1, device=dev, dtype=i32)
        # RBD plan
        self.has_rbd = s.rbd_epd is not None and s.rbd_dpn is not None
        if self.has_rbd:
            epn = s.rbd_epd * s.rbd_dpn
            self.n_nodes = E // epn
            pmax = T * min(k, self.n_nodes)
            self.pilots_per_node = e(self.n_nodes, dtype=i32)
            self.node_offsets = e(self.n_nodes + 1, dtype=i32)
            self.pilot_token = e(max(pmax, 1), dtype=i32)
            self.pilot_node = e(max(pmax, 1), dtype=i32)
            self.pilot_device = e(max(pmax, 1), dtype=i32)
            self.replica_offsets = e(pmax + 1, dtype=i32)
            self.replica_expert = e(max(N, 1), dtype=i32)
            self.assign_pilot = e(T, k, dtype=i32)
            self.rbd_counts = e(2, dtype=i32)
            self.rbd_ws_bytes = L.rbd_plan_workspace_size(T, k, E, s.rbd_epd, s.rbd_dpn)
            self.rbd_ws = e(max(self.rbd_ws_bytes, 256), dtype=torch.uint8)
            # The RBD plan reads only the routing ids, so step() runs it on a side stream next
            # to dispatch / experts / backward; these events fork it after routing and join it
            # back before the step ends (so the next step's routing cannot overwrite ids in use).
            if self.device.type == "cuda":
                self.side = torch.cuda.Stream(device=self.device)
                self.ev_routed = torch.cuda.Event()
                self.ev_rbd_done = torch.cuda.Event()

    # ------------------------------------------------------------------ steps
    def route(self, x, wg, bias=None, stream=None):
        s = self.s
        L.moe_route(x, wg, bias, s.T, s.d, s.E, s.k, self.code, self.logits, self.topk_ids, self.topk_w,
                    self.route_ws, self.route_ws_bytes, self.err, stream)

    def build_pft(self, stream=None):
        s = self.s
        L.pft_build(self.topk_ids, self.topk_w, s.T, s.E, s.k, self.tokens_per_expert, self.expert_offsets,
                    self.token_ids, self.expert_ids, self.combine_weights, self.pos, self.tile_offsets, self.pft_ws,
                    self.pft_ws_bytes, self.err, stream)

    def dispatch(self, x, stream=None):
        s = self.s
        L.moe_dispatch(x, self.pos, s.T, s.k, s.d, self.code, self.x_pft, self.err, stream)

    def experts(self, w1, w3, w2, stream=None):
        s = self.s
        L.moe_expert_ffn(self.x_pft, self.expert_offsets, self.tile_offsets, s.N, s.E, s.d, s.h, self.code, w1, w3,
                         w2, self.h1, self.h3, self.a, self.out, self.err, stream)

    def experts_gathered(self, x, w1, w3, w2, stream=None):
        s = self.s
        L.moe_expert_ffn_gathered(x, self.token_ids, self.expert_offsets, self.tile_offsets, s.N, s.E, s.d, s.h,
                                  self.code, w1, w3, w2, self.h1, self.h3, self.a, self.out, self.err, stream)

    def combine(self, stream=None):
        s = self.s
        L.moe_combine(self.out, self.pos, self.topk_w, s.T, s.k, s.d, self.code, self.y, self.err, stream)

    def forward(self, x, wg, bias, w1, w3, w2, stream=None):
        self.route(x, wg, bias, stream)
        self.build_pft(stream)
        if self.fused_gather:
            self.experts_gathered(x, w1, w3, w2, stream)
        else:
            self.dispatch(x, stream)
            self.experts(w1, w3, w2, stream)
        self.combine(stream)
        return self.y

    def backward(self, dy, x, wg, w1, w3, w2, stream=None):
        s = self.s
        if self.fused_gather:
            self.dispatch(x, stream)   # the PFT copy of x, for the weight gradients only
        L.moe_backward(dy, x, wg, self.topk_w, self.topk_ids, self.pos, self.expert_offsets, self.tile_offsets,
                       self.x_pft, self.h1, self.h3, self.a, self.out, w1, w3, w2, s.T, s.d, s.E, s.h, s.k, self.code,
                       self.dx, self.dwg, self.dw1, self.dw3, self.dw2, self.dlogits, self.bwd_ws, self.bwd_ws_bytes,
                       self.err, stream)
        return self.dx

    def rbd(self, stream=None):
        s = self.s
        if not self.has_rbd:
            raise ValueError("this layer shape has no RBD device map")
        L.rbd_plan(self.topk_ids, s.T, s.k, s.E, s.rbd_epd, s.rbd_dpn, self.pilots_per_node, self.node_offsets,
                   self.pilot_token, self.pilot_node, self.pilot_device, self.replica_offsets, self.replica_expert,
                   self.assign_pilot, self.rbd_counts, self.rbd_ws, self.rbd_ws_bytes, self.err, stream)

    def step(self, x, wg, bias, w1, w3, w2, dy, stream=None, overlap_rbd=True):
        """One pass of the whole hot path: forward, RBD plan (if mapped), backward.

        With an RBD map the plan runs on a side stream forked after routing and joined
        before return, overlapping the PFT build, the expert GEMMs and the backward
        (overlap_rbd=False runs it in line after routing instead)."""
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.route(x, wg, bias, main)
        if self.has_rbd and not overlap_rbd:
            self.rbd(main)
        elif self.has_rbd:
            self.ev_routed.record(main)
            self.side.wait_event(self.ev_routed)
            self.rbd(self.side)
            self.ev_rbd_done.record(self.side)
        self.build_pft(main)
        if self.fused_gather:
            self.experts_gathered(x, w1, w3, w2, main)
        else:
            self.dispatch(x, main)
            self.experts(w1, w3, w2, main)
        self.combine(main)
        self.backward(dy, x, wg, w1, w3, w2, main)
        if self.has_rbd and overlap_rbd:
            main.wait_event(self.ev_rbd_done)

    def device_error(self) -> int:
        """Read (synchronously) and return the device error word; 0 means no device-side fault."""
        return int(self.err.item())
