"""MoE MLP block of both flows with router replay, composed from library calls.

Page "Sintesi Tecnica: Dual-Flow Transformers", section "Meccanismi Chiave"
(router replay) and section "Contributi Chiave" (independent expert fan-outs
of the two flows). One block call: route (primary top-k_aux, gates of both
flows) -> dispatch (each expert's rows packed into a fixed [128][d] block) ->
the gate/up projections of all experts in one batched launch (SwiGLU
epilogue), then the down projections of all experts in one batched launch,
each hinting the other's weights into L2 -> combine (+ residual). Every
expert's weights stream from HBM once per call for both flows.
"""

from __future__ import annotations

import torch

from . import api


class DualFlowMoE:
    def __init__(self, w_router, w_gu, w_down, k, k_aux=None, B=64, device="cuda"):
        """w_router bf16 [E, d]; w_gu bf16 [E, 2F, d] ([W_gate; W_up] per
        expert); w_down bf16 [E, d, F]; B tokens per flow (<= 64)."""
        if B > api.MOE_ROWS:
            raise ValueError("at most %d tokens per flow per call" % api.MOE_ROWS)
        E, d = w_router.shape
        self.E, self.d, self.F = E, d, w_gu.shape[1] // 2
        self.k = k
        self.k_aux = k if k_aux is None else k_aux
        self.B = B
        self.w_router, self.w_gu, self.w_down = w_router, w_gu, w_down
        dev = torch.device(device)
        rows = 2 * api.MOE_ROWS
        self.xe = torch.zeros((E, rows, d), dtype=torch.bfloat16, device=dev)
        self.h = torch.empty((E, rows, self.F), dtype=torch.bfloat16, device=dev)
        self.ye = torch.zeros((E, rows, d), dtype=torch.bfloat16, device=dev)
        self.ids = torch.empty((B, self.k_aux), dtype=torch.int32, device=dev)
        self.g1 = torch.empty((B, self.k), dtype=torch.float32, device=dev)
        self.g2 = torch.empty((B, self.k_aux), dtype=torch.float32, device=dev)
        self.slot1 = torch.empty((B, self.k), dtype=torch.int32, device=dev)
        self.slot2 = torch.empty((B, self.k_aux), dtype=torch.int32, device=dev)
        self.counts = torch.zeros((E, 2), dtype=torch.int32, device=dev)
        self.y = torch.empty((2 * B, d), dtype=torch.bfloat16, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        ws = max(api.grouped_proj_workspace_size(rows, 2 * self.F, d, "swiglu"),
                 api.grouped_proj_workspace_size(rows, d, self.F, "none"))
        self.ws = torch.zeros(max(256, ws), dtype=torch.uint8, device=dev)
        self.launches = 3 + (api.grouped_proj_batched_num_launches(rows, 2 * self.F, d, "swiglu", E)
                             + api.grouped_proj_batched_num_launches(rows, d, self.F, "none", E))

    def forward(self, x, residual=None, stream=None):
        """x: bf16 [2B, d] (primary rows, then auxiliary rows). Returns the
        block output [2B, d] (a preallocated buffer)."""
        B, E = self.B, self.E
        api.moe_route(x, B, self.w_router, self.k, self.k_aux, ids=self.ids, g1=self.g1,
                      g2=self.g2, stream=stream)
        api.moe_dispatch(x, B, self.ids, E, self.k, self.k_aux, xe=self.xe, slot1=self.slot1,
                         slot2=self.slot2, counts=self.counts, err_flag=self.err, stream=stream)
        self.experts(stream)
        return api.moe_combine(self.ye, self.ids, self.g1, self.g2, self.slot1, self.slot2, B,
                               self.k, self.k_aux, residual=residual, y=self.y,
                               err_flag=self.err, stream=stream)

    def experts(self, stream=None):
        """The experts' SwiGLU MLPs: all gate/up projections in one batched
        launch, then all down projections (each hinting the other's weights,
        the down launch the next call's gate/up)."""
        api.grouped_proj_batched(self.xe, api.MOE_ROWS, self.w_gu, y=self.h, epilogue="swiglu",
                                 workspace=self.ws, err_flag=self.err, stream=stream,
                                 next_w=self.w_down, next_epilogue="none")
        api.grouped_proj_batched(self.h, api.MOE_ROWS, self.w_down, y=self.ye, workspace=self.ws,
                                 err_flag=self.err, stream=stream, next_w=self.w_gu,
                                 next_epilogue="swiglu")
