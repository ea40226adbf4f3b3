"""One Dual-Flow decoder layer at one generated position, both flows.

Composition of library calls only (each step is a libdualflow kernel):

  1. RMSNorm of X = [x1 rows; x2 rows]                      dualflow_rmsnorm
  2. QKV = Xn W_qkv^T, one GEMM for both flows; auxiliary
     rows stored only for the Q columns                       dualflow_grouped_proj
  3. append the primary rows' K/V at position L (the
     auxiliary flow never writes the cache)                  dualflow_kv_append
  4. dual decode attention over L + 1 tokens, Q2 coupled
     to Q1 through a_l inside the kernel                     dualflow_decode_attn
  5. X' = X + O W_o^T                                        dualflow_grouped_proj (residual)
  6. RMSNorm of X'                                           dualflow_rmsnorm
  7. H = SiLU(X'n W_gate^T) * (X'n W_up^T), aux += b_l H1    dualflow_grouped_proj (swiglu)
  8. X'' = X' + H W_down^T, aux += c_l (H1 W_down^T)         dualflow_grouped_proj (residual)

By default (fused_pre=True) steps 1-3 run as one launch
(dualflow_layer_pre_attention) when the sizes allow it: 4-CTA clusters split
the QKV product along K and reduce it through distributed shared memory, the
first norm's row scale multiplies the accumulator (the normalised rows are
not stored) and the primary K/V columns go straight into the cache.
fused_pre=False, or sizes the fused launch does not take, use the three calls.
With split_pre=True (the default) the fused pre-attention launch stops short
of the reduction (dualflow_layer_qkv_partials: fp32 partial products of the
4 quarters of K and their row sums of squares) and the attention launch
(dualflow_decode_attn_qkv_partials) sums, scales and rounds its KV head's
query rows and appends the primary K/V row in its prologue: the same bits as
the fused launch followed by dualflow_decode_attn, without the reduction's
round trip between the cluster's shared memories on the critical path.

By default (fused_post=True) steps 5-8 run as one persistent launch
(dualflow_layer_post_attention) when the sizes allow it: its weight producers
stream W_o, W_gate/up and W_down back to back instead of four launches each
ramping up and draining, the W_o and W_down split-k sums are reduced inside
4-CTA clusters, and the norm's row scale multiplies the gate/up accumulators
(the normalised rows are not stored). fused_post=False, or sizes the fused
launch does not take, use the four calls.

Pages: "Sintesi Tecnica: Dual-Flow Transformers", sections "Architettura
Core" (shared matrices, primary-only cache writes, auxiliary flow active at
generated positions), "Meccanismi Chiave" (asymmetric shared-KV attention and
the a/b/c coupling vectors) and "Costi di Inferenza" (grouped decode reads the
weights and the cache once for both flows). The normalisation, SwiGLU MLP and
the additive coupling forms are the readings taken where the pages are silent.
"""

from __future__ import annotations

import torch

from . import api


class DualFlowLayer:
    def __init__(self, weights, Hq, Hkv, D, F, B, max_seqlen, device="cuda", eps=1e-5,
                 num_splits=0, fused_pre=True, fused_post=True, split_pre=True,
                 layer_stack=False):
        self.w = weights  # dict of device tensors: w_qkv, w_o, w_gu, w_down, a, b, c
        self.Hq, self.Hkv, self.D, self.F, self.B = Hq, Hkv, D, F, B
        self.d_model = weights["w_o"].shape[0]
        self.max_seqlen = int(max_seqlen)
        self.eps = eps
        self.num_splits = num_splits
        dev = torch.device(device)
        bf = torch.bfloat16
        M = 2 * B
        qd, kvd = Hq * D, Hkv * D
        self.xn = torch.empty(M, self.d_model, dtype=bf, device=dev)
        self.qkv = torch.empty(M, qd + 2 * kvd, dtype=bf, device=dev)
        self.attn = torch.empty(M, qd, dtype=bf, device=dev)
        self.x_mid = torch.empty(M, self.d_model, dtype=bf, device=dev)
        self.xn2 = torch.empty(M, self.d_model, dtype=bf, device=dev)
        self.h = torch.empty(M, F, dtype=bf, device=dev)
        self.x_out = torch.empty(M, self.d_model, dtype=bf, device=dev)
        self.x_in = torch.empty(M, self.d_model, dtype=bf, device=dev)
        ws = max(api.grouped_proj_workspace_size(M, *weights["w_qkv"].shape, "none"),
                 api.grouped_proj_workspace_size(M, *weights["w_o"].shape, "residual"),
                 api.grouped_proj_workspace_size(M, *weights["w_gu"].shape, "swiglu"),
                 api.grouped_proj_workspace_size(M, *weights["w_down"].shape, "residual"))
        self.proj_ws = torch.zeros(ws, dtype=torch.uint8, device=dev)
        self.attn_ws = api.new_attn_workspace(B, Hq, Hkv, D, self.max_seqlen, num_splits, dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.attn_launches = api.decode_attn_num_launches(B, Hkv, self.max_seqlen, num_splits)
        self.fused_pre = bool(fused_pre) and \
            api.layer_pre_attention_supported(B, self.d_model, Hq, Hkv, D)
        self.split_pre = self.fused_pre and bool(split_pre)
        self.qkv_part = (torch.empty(4, M, qd + 2 * kvd, dtype=torch.float32, device=dev)
                         if self.split_pre else None)
        self.ss_part = (torch.empty(4, M, dtype=torch.float32, device=dev)
                        if self.split_pre else None)
        self.fused_post = bool(fused_post) and \
            api.layer_post_attention_workspace_size(B, self.d_model, qd, F) > 0
        self.post_ws = (api.new_post_attention_workspace(B, self.d_model, qd, F, dev)
                        if self.fused_post else None)
        if self.fused_post:
            post_launches = 1
        else:
            post_launches = (api.grouped_proj_num_launches(M, *weights["w_o"].shape, "residual")
                             + 1
                             + api.grouped_proj_num_launches(M, *weights["w_gu"].shape, "swiglu")
                             + api.grouped_proj_num_launches(M, *weights["w_down"].shape,
                                                             "residual"))
        pre_launches = 1 if self.fused_pre else \
            2 + api.grouped_proj_num_launches(M, *weights["w_qkv"].shape, "none")
        self._launches = pre_launches + self.attn_launches + post_launches
        # Layer-stack form of the captured step: the post-attention launch
        # also computes the NEXT step's QKV partial products from x_out, as
        # in a stack of layers where each output is the next one's input;
        # captured steps then alternate between two buffers (x_in -> x_alt
        # -> x_in ...), one launch fewer per step.
        self.layer_stack = bool(layer_stack)
        if self.layer_stack:
            if not (self.split_pre and self.fused_post):
                raise ValueError("the layer-stack form needs the split pre-attention and the "
                                 "fused post-attention launches")
            self.x_alt = torch.empty(M, self.d_model, dtype=bf, device=dev)
            self._launches = self.attn_launches + 1

    @property
    def launches_per_step(self) -> int:
        """Kernel launches of one step: the pre-attention half (one launch
        fused, else the first norm, the QKV projection and the append), the
        attention and the post-attention half (one launch fused, else W_o, the
        second norm, gate/up and down)."""
        return self._launches

    # ------------------------------------------------------------ CUDA graphs
    def capture(self, X, k_cache, v_cache, block_table, positions, seqlens):
        """Capture the step over fixed buffers as one CUDA graph (one launch
        per step; consecutive kernels keep their programmatic-dependent-launch
        overlap) and, for timing the attention alone, as three graphs (before
        attention, attention, after attention) with events between them. The
        step runs once eagerly first, so one-time host set-up happens outside
        the captures."""
        args = (X, k_cache, v_cache, block_table, positions, seqlens)
        self.step(*args)
        torch.cuda.synchronize()
        self._graph_args = args
        self.graph_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_full):
            for part in ("pre", "attn", "post"):
                self._step_part(part, *args)
        self.graphs = []
        for part in ("pre", "attn", "post"):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._step_part(part, *args)
            self.graphs.append(g)
        torch.cuda.synchronize()
        if self.layer_stack:
            # the partials of X, then one eager step each way; two graphs
            # (X -> x_alt, x_alt -> X), and for the timers the attention and
            # the post-attention launch X -> x_alt
            w = self.w
            x_save = X.clone()
            api.layer_qkv_partials(X, w["w_qkv"], self.Hq, self.Hkv, self.D, part=self.qkv_part,
                                   ss_part=self.ss_part, err_flag=self.err)
            self._stack_step(X, self.x_alt, args)
            self._stack_step(self.x_alt, X, args)
            torch.cuda.synchronize()
            self.stack_graphs = []
            for src, dst in ((X, self.x_alt), (self.x_alt, X)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    self._stack_step(src, dst, args)
                self.stack_graphs.append(g)
            self.stack_post = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.stack_post):
                self._stack_post(X, self.x_alt)
            # back to X and its partials: the first replay is the step on X
            X.copy_(x_save)
            api.layer_qkv_partials(X, w["w_qkv"], self.Hq, self.Hkv, self.D, part=self.qkv_part,
                                   ss_part=self.ss_part, err_flag=self.err)
            self._stack_next = 0
            torch.cuda.synchronize()

    def _stack_post(self, X, x_out, stream=None):
        w = self.w
        api.layer_post_attention(self.attn, X, w["w_o"], w["w_gu"], w["w_down"], w["b"], w["c"],
                                 eps=self.eps, x_mid=self.x_mid, h=self.h, x_out=x_out,
                                 workspace=self.post_ws, err_flag=self.err, stream=stream,
                                 qkv_next=(w["w_qkv"], self.Hq, self.Hkv, self.D,
                                           self.qkv_part, self.ss_part))

    def _stack_step(self, X, x_out, args, stream=None):
        """Layer-stack step: attention over the partials the previous step
        left, then the post-attention launch X -> x_out with the next QKV."""
        self._step_part("attn", *args, stream=stream)
        self._stack_post(X, x_out, stream=stream)

    def replay(self, timers=None):
        """One captured step on the current stream: the single-graph step, or
        with timers ({"attn": (start_event, end_event)}) the three-graph step
        with the events recorded around the attention. In the layer-stack form
        the steps alternate X -> x_alt -> X ... (each step's input is the
        previous output; returns the buffer just written); with timers, the
        attention and the post-attention launch X -> x_alt."""
        if self.layer_stack:
            if timers is None:
                i = self._stack_next
                self.stack_graphs[i].replay()
                self._stack_next = 1 - i
                return self.x_alt if i == 0 else self._graph_args[0]
            timers["attn"][0].record()
            self.graphs[1].replay()
            timers["attn"][1].record()
            self.stack_post.replay()
            return self.x_alt
        if timers is None:
            self.graph_full.replay()
            return self.x_out
        self.graphs[0].replay()
        timers["attn"][0].record()
        self.graphs[1].replay()
        timers["attn"][1].record()
        self.graphs[2].replay()
        return self.x_out

    def step(self, X, k_cache, v_cache, block_table, positions, seqlens, stream=None,
             timers=None):
        """X: bf16 [2B, d_model] (primary rows then auxiliary rows). Returns the
        layer output (a preallocated buffer, overwritten by the next step).
        seqlens must equal positions + 1 (the attended length after the append).
        timers: optional dict of (start, end) CUDA events around the attention."""
        args = (X, k_cache, v_cache, block_table, positions, seqlens)
        self._step_part("pre", *args, stream=stream)
        if timers is not None:
            timers["attn"][0].record()
        self._step_part("attn", *args, stream=stream)
        if timers is not None:
            timers["attn"][1].record()
        self._step_part("post", *args, stream=stream)
        return self.x_out

    def _step_part(self, part, X, k_cache, v_cache, block_table, positions, seqlens, stream=None):
        """One third of the step: "pre" (norm, QKV, append), "attn", "post"."""
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        qd, kvd = Hq * D, Hkv * D
        w = self.w
        qkv = self.qkv
        # Each projection warms L2 with the first weight blocks of the next one
        # (o -> gate/up -> down -> the next step's QKV); none after the QKV
        # projection, whose successor is the HBM-bound attention.
        if part == "pre" and self.split_pre:
            api.layer_qkv_partials(X, w["w_qkv"], Hq, Hkv, D, part=self.qkv_part,
                                   ss_part=self.ss_part, err_flag=self.err, stream=stream)
        elif part == "pre" and self.fused_pre:
            api.layer_pre_attention(X, w["w_qkv"], Hq, Hkv, k_cache, v_cache, block_table,
                                    positions, eps=self.eps, qkv=qkv, err_flag=self.err,
                                    stream=stream)
        elif part == "pre":
            api.rmsnorm(X, y=self.xn, eps=self.eps, stream=stream)
            api.grouped_proj(self.xn, B, w["w_qkv"], n_aux=qd, y=qkv, workspace=self.proj_ws,
                             err_flag=self.err, stream=stream)
            api.kv_append(qkv[:B, qd:qd + kvd].view(B, Hkv, D), qkv[:B, qd + kvd:].view(B, Hkv, D),
                          k_cache, v_cache, block_table, positions, err_flag=self.err,
                          stream=stream)
        elif part == "attn" and self.split_pre:
            api.decode_attn_qkv_partials(
                self.qkv_part, self.ss_part, self.d_model, w["a"], k_cache, v_cache, block_table,
                seqlens, self.max_seqlen, Hq, eps=self.eps, o1=self.attn[:B].view(B, Hq, D),
                o2=self.attn[B:].view(B, Hq, D), num_splits=self.num_splits,
                workspace=self.attn_ws, err_flag=self.err, stream=stream)
        elif part == "attn":
            api.decode_attn(qkv[:B, :qd].view(B, Hq, D), qkv[B:, :qd].view(B, Hq, D), w["a"],
                            k_cache, v_cache, block_table, seqlens, self.max_seqlen,
                            o1=self.attn[:B].view(B, Hq, D), o2=self.attn[B:].view(B, Hq, D),
                            num_splits=self.num_splits, workspace=self.attn_ws,
                            err_flag=self.err, stream=stream)
        elif self.fused_post:
            api.layer_post_attention(self.attn, X, w["w_o"], w["w_gu"], w["w_down"], w["b"],
                                     w["c"], eps=self.eps, x_mid=self.x_mid, h=self.h,
                                     x_out=self.x_out, workspace=self.post_ws,
                                     err_flag=self.err, stream=stream)
        else:
            api.grouped_proj(self.attn, B, w["w_o"], y=self.x_mid, epilogue="residual",
                             residual=X, workspace=self.proj_ws, err_flag=self.err,
                             stream=stream, next_w=w["w_gu"], next_epilogue="swiglu")
            api.rmsnorm(self.x_mid, y=self.xn2, eps=self.eps, stream=stream)
            api.grouped_proj(self.xn2, B, w["w_gu"], y=self.h, epilogue="swiglu",
                             coupling=w["b"], workspace=self.proj_ws, err_flag=self.err,
                             stream=stream, next_w=w["w_down"], next_epilogue="residual")
            api.grouped_proj(self.h, B, w["w_down"], y=self.x_out, epilogue="residual",
                             coupling=w["c"], residual=self.x_mid, workspace=self.proj_ws,
                             err_flag=self.err, stream=stream, next_w=w["w_qkv"],
                             next_epilogue="none")


    def step_host(self, x_host, out_host, k_cache, v_cache, block_table, positions, seqlens,
                  stream=None):
        """Host-buffer entry point: copies X from (pinned) host memory, runs the
        step and copies the layer output back, all queued on the stream."""
        self.x_in.copy_(x_host, non_blocking=True)
        if getattr(self, "graphs", None) and self._graph_args[0] is self.x_in:
            # (a new input has no partials from a previous step: the whole
            # three-launch step, also in the layer-stack form)
            self.graph_full.replay()
            out = self.x_out
        else:
            out = self.step(self.x_in, k_cache, v_cache, block_table, positions, seqlens,
                            stream=stream)
        out_host.copy_(out, non_blocking=True)
        return out_host
