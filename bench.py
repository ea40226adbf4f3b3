#!/usr/bin/env python
"""Benchmark of the Dual-Flow decode step on B200.

One step = one Dual-Flow decoder layer at one generated position for a batch
of sequences, both flows: RMSNorm, grouped QKV projection (both flows' rows,
one tcgen05 GEMM), primary-only KV append, dual shared-KV decode attention
(split + combine), grouped W_o projection with residual, RMSNorm, grouped
gate/up projection with fused SwiGLU + b coupling, grouped down projection
with residual + c coupling. Default workload: d_model 4096, 32 query heads
per flow on 8 KV heads, head_dim 128, SwiGLU width 14336, 64 sequences per
flow (M = 128 rows), cache 4096 tokens + the appended one, bf16 weights
~ N(0, 0.02), synthetic seeded data. Metric: decode tokens/s (one token per
sequence per step, per layer) and the KV-read GB/s of the attention kernel.

--impl reference times the fp64 CPU oracle on the machine's host cores on a
bounded sample of the same workload (the reference arm for this method has no
upstream code to run).

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
sequences with its own cache and weight replica (weak scaling; sequences are
independent, so there is no data-path collective); the timed region is
bracketed by barriers and the slowest rank's time is reported.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dual-flow decode tokens/s and KV-read GB/s (% of B200 HBM peak), 1 GPU"
PREFILL_METRIC = ("primary prefill prompt tokens/s (one layer's causal attention, cache write "
                  "and last-position auxiliary query), 1 GPU")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, NVIDIA's nominal figure
FALLBACK_BF16_TFLOPS = 1590.0
CSRC = os.path.join(ROOT, "dual_flow_transformer_b200", "csrc")
ATTN_SRC = os.path.join(CSRC, "decode_attn.cu")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload",
                    choices=["layer", "mha", "gqa", "long", "tiny", "mixture", "moe",
                             "prefill"],
                    default="layer")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--fused-pre", type=int, choices=[0, 1], default=None,
                    help="layer workload: 1 = norm, QKV and the append as one launch, "
                         "0 = three launches (default: the layer's own default)")
    ap.add_argument("--split-pre", type=int, choices=[0, 1], default=None,
                    help="layer workload, with the one-launch pre-attention half: 1 = it "
                         "stores fp32 partial products that the attention launch reduces, "
                         "0 = it reduces them itself (default: the layer's own default)")
    ap.add_argument("--layer-stack", action="store_true",
                    help="layer workload: time the layer-stack form (the post-attention launch "
                         "also computes the next step's QKV partial products; each step's input "
                         "is the previous step's output)")
    ap.add_argument("--fused-post", type=int, choices=[0, 1], default=None,
                    help="layer workload: 1 = the post-attention half as one persistent launch, "
                         "0 = four launches (default: the layer's own default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0,
                    help="target seconds of oracle work for the CPU baseline sample")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers

def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor-core peak: the burst cuBLAS figure (a kernel timed on
    its own), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["bf16_tflops"])
        return v, "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def traffic_from_profile(workload, prefix="decode_attn", src=ATTN_SRC):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when there is none or the kernel source changed since it
    was captured."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (prefix, workload))
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != sha:
        return None
    try:
        return int(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


_SAMPLER_SRC = r"""
import sys, time
import pynvml as N
pynvml_bus, idx, out = sys.argv[1], int(sys.argv[2]), open(sys.argv[3], "w")
N.nvmlInit()
try:
    h = N.nvmlDeviceGetHandleByPciBusId(pynvml_bus) if pynvml_bus else N.nvmlDeviceGetHandleByIndex(idx)
except Exception:
    h = N.nvmlDeviceGetHandleByIndex(idx)
smax = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
print("ready %d" % smax, flush=True)
while True:
    t = time.time()
    sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
    try:
        r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
    except Exception:
        r = N.nvmlDeviceGetCurrentClocksThrottleReasons(h)
    out.write("%.6f %d %d\n" % (t, sm, r))
    out.flush()
    time.sleep(0.0005)
"""

# NVML clock-event reason bits (nvml.h)
_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


class ClockSampler:
    """SM clock and clock-event reasons sampled by NVML every ~0.5 ms (each
    sample is two read-only queries) from a separate process into a file,
    kept only for the host-time window that brackets the timed GPU work
    (start() ... stop())."""

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.smax = None
        self.t0 = self.t1 = None

    def start(self):
        import torch
        bus = ""
        try:
            pr = torch.cuda.get_device_properties(self.device)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        except Exception:
            pass
        idx = self.device.index or 0
        try:
            # samples go to a file (a pipe left unread would fill and stall the sampler)
            fd, self.path = tempfile.mkstemp(suffix=".clk")
            os.close(fd)
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_SRC, bus, str(idx),
                                          self.path],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            line = self.proc.stdout.readline().split()
            self.smax = float(line[1]) if len(line) == 2 and line[0] == "ready" else None
            if self.smax is None:
                self.proc.kill()
                self.proc = None
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        """{"sm_mhz": median, "sm_max_mhz", "reasons", "samples", "window_ms"}
        over the timed window, or a record saying why there is none."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML sampler unavailable"}
        self.proc.kill()
        self.proc.communicate(timeout=10)
        with open(self.path) as f:
            out = f.read()
        os.unlink(self.path)
        sm, reasons = [], set()
        for row in out.splitlines():
            f = row.split()
            try:
                t, mhz, bits = float(f[0]), float(f[1]), int(f[2])
            except (IndexError, ValueError):
                continue
            if self.t0 is None or self.t1 is None or not (self.t0 <= t <= self.t1):
                continue
            sm.append(mhz)
            for name, bit in _REASON_BITS.items():
                if bits & bit:
                    reasons.add(name)
        rec = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
               "reasons": sorted(reasons), "samples": len(sm),
               "window_ms": None if self.t0 is None else round((self.t1 - self.t0) * 1e3, 2),
               "how": "NVML queries every ~0.5 ms from a separate process, host-time window "
                      "around the timed passes"}
        if not sm:
            rec["note"] = "no sample fell inside the timed window"
        return rec


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(value, world, device="cuda"):
    """Slowest rank's value (timing plumbing, not a data-path collective)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base, rank):
    """Weak scaling: every rank decodes its own batch of sequences."""
    return base + 1000 * rank


def workload_config(name, w, host, world=1):
    """The workload as both arms name it in their JSON lines: its sizes and
    whether its inputs exceed L2, from the workload and its host inputs alone
    (no device, no library). How this build runs it goes under "path"."""
    if name == "layer":
        L = w.cache_len + 1
        kv = w.B * L * w.Hkv * w.D * 2 * 2
        cfg = {"workload": "dual-flow decoder layer step: d_model %d, %d/%d heads, head_dim %d, "
                           "SwiGLU %d, batch %d per flow (M=%d), cache %d+1"
                           % (w.d_model, w.Hq, w.Hkv, w.D, w.F, w.B, 2 * w.B, w.cache_len),
               "batch_per_flow": w.B, "rows": 2 * w.B, "cache_len": w.cache_len,
               "attended": L,
               "l2": "inputs larger than L2 (KV %.2f GB + weights %.2f GB read per step)"
                     % (kv / 1e9, 436207616 / 1e9)}
    elif name == "mixture":
        B, V, d = w.B, w.V, w.d_model
        cfg = {"workload": "dual-flow mixture head: LM-head projection of both flows (batch %d "
                           "per flow, M=%d, d_model %d, vocabulary %d, bf16 weights %.1f MB) + "
                           "mixed next-token distribution (fp32)"
                           % (B, 2 * B, d, V, V * d * 2 / 1e6),
               "l2": "inputs larger than L2 (%.0f MB of weights per step)" % (V * d * 2 / 1e6)}
    elif name == "moe":
        B, d, F, E = w.B, w.d_model, w.F, w.E
        cfg = {"workload": "dual-flow MoE MLP block with router replay: %d tokens per flow, "
                           "d_model %d, %d SwiGLU experts of width %d, primary top-%d, auxiliary "
                           "fan-out %d (%.1f MB of expert weights)"
                           % (B, d, E, F, w.k, w.k_aux, E * 3 * F * d * 2 / 1e6),
               "l2": "inputs larger than L2 (%.0f MB of expert weights per step)"
                     % (E * 3 * F * d * 2 / 1e6)}
    elif name == "prefill":
        cfg = {"workload": "dual-flow primary prefill: %d fresh prompts of %d..%d tokens, %d/%d "
                           "heads, head_dim %d, bf16, 64-token pages in a random block table, "
                           "auxiliary query at each last position"
                           % (host["B"], w.len_lo, w.len_hi, w.Hq, w.Hkv, w.D),
               "l2": "inputs larger than L2 (%.0f MB of queries, %.0f MB of new K/V)"
                     % (host["q1"].numel() * 2 / 1e6, 2 * host["k_new"].numel() * 2 / 1e6)}
    else:
        esize = 4 if w.dtype == "fp32" else 2
        kv = int(host["seqlens"].sum()) * w.Hkv * w.D * 2 * esize
        cfg = {"workload": "dual-flow decode attention '%s': batch %d, %d/%d heads, head_dim %d, "
                           "%s, lengths %d..%d%s" % (
                               name, w.B, w.Hq, w.Hkv, w.D, w.dtype, w.len_lo, w.len_hi,
                               ", random block table" if w.random_table else ""),
               "l2": "inputs larger than L2" if kv > 126e6
                     else "inputs smaller than L2 (not flushed)"}
    cfg["parallelism"] = "replicas" if world > 1 else "single GPU"
    return cfg


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- workloads

def attn_algorithmic_bytes(B, Hq, Hkv, D, seqlens_sum, esize, dual=True):
    """Per decode-attention launch: K and V read once + Q1 (+ Q2raw, a) + O1 (+ O2)."""
    kv = seqlens_sum * Hkv * D * 2 * esize
    q = B * Hq * D * esize * (2 if dual else 1)
    a = Hq * D * esize if dual else 0
    o = B * Hq * D * esize * (2 if dual else 1)
    return kv + q + a + o


class LayerRun:
    """The full layer step of the 'layer' workload on this GPU."""

    def __init__(self, args, dev, seed):
        import torch
        from dual_flow_transformer_b200 import synth
        from dual_flow_transformer_b200.layer import DualFlowLayer
        w = synth.WORKLOADS["layer"]
        self.w = w
        self.host = synth.make_layer_inputs(w, seed=seed)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.host.items()}
        self.d = d
        W = {k: d[k] for k in ("w_qkv", "w_o", "w_gu", "w_down", "a", "b", "c")}
        kw = {} if args.fused_post is None else {"fused_post": bool(args.fused_post)}
        if args.fused_pre is not None:
            kw["fused_pre"] = bool(args.fused_pre)
        if args.split_pre is not None:
            kw["split_pre"] = bool(args.split_pre)
        if args.layer_stack:
            kw["layer_stack"] = True
        self.layer = DualFlowLayer(W, w.Hq, w.Hkv, w.D, w.F, w.B, w.cache_len + 1, device=dev,
                                   num_splits=args.num_splits, **kw)
        self.X = torch.cat([d["x1"], d["x2"]]).contiguous()
        self.seqlens = (d["positions"] + 1).to(torch.int32)
        # the step runs as CUDA-graph replays over fixed buffers (X lives in x_in)
        self.layer.x_in.copy_(self.X)
        self.layer.capture(self.layer.x_in, d["k_cache"], d["v_cache"], d["block_table"],
                           d["positions"], self.seqlens)
        self.tokens_per_step = w.B
        self.launches_per_step = self.layer.launches_per_step
        L = w.cache_len + 1
        self.attn_bytes = attn_algorithmic_bytes(w.B, w.Hq, w.Hkv, w.D, w.B * L, 2)
        self.kv_bytes = w.B * L * w.Hkv * w.D * 2 * 2
        self.units = w.B * w.Hkv * L  # (sequence, KV head, token) units per attention launch
        self.bytes_per_unit = w.D * 2 * 2
        self.config = workload_config("layer", w, self.host)
        self.path = {"attn_launches": self.layer.attn_launches,
                     "pre_attention": ("one launch, reduced in the attention launch"
                                       if self.layer.split_pre else "one launch")
                                      if self.layer.fused_pre else "three launches",
                     "post_attention": "one persistent launch" if self.layer.fused_post
                                       else "four launches"}
        if self.layer.layer_stack:
            self.path["pre_attention"] = ("inside the previous step's post-attention launch "
                                          "(layer-stack form: each step's input is the previous "
                                          "step's output; e2e runs the three-launch step)")
        self.dominant = "dualflow_decode_attn (split kernel, combine inside it)"

    def step(self, timers=None):
        self.layer.replay(timers)

    def attn_graphs(self):
        """(dual attention graph, primary-only attention graph) on this step's
        buffers: the same call with q2raw = NULL writes O1 only."""
        import torch
        from dual_flow_transformer_b200 import api
        L, d = self.layer, self.d
        B, Hq, D = L.B, L.Hq, L.D
        o1 = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=L.qkv.device)

        def call():
            api.decode_attn(L.qkv[:B, :Hq * D].view(B, Hq, D), None, None, d["k_cache"],
                            d["v_cache"], d["block_table"], self.seqlens, L.max_seqlen, o1=o1,
                            num_splits=L.num_splits, workspace=L.attn_ws, err_flag=L.err)
        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        self._primary_o1 = o1
        return L.graphs[1], g

    def step_host(self, x_host, out_host):
        d = self.d
        self.layer.step_host(x_host, out_host, d["k_cache"], d["v_cache"], d["block_table"],
                             d["positions"], self.seqlens)

    def host_io(self):
        import torch
        xh = torch.cat([self.host["x1"], self.host["x2"]]).contiguous().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        return xh, oh

    def check_err(self):
        return int(self.layer.err.item())


class AttnRun:
    """Decode attention alone on one of the attention workloads."""

    def __init__(self, args, dev, seed, name):
        import torch
        from dual_flow_transformer_b200 import api, synth
        w = synth.WORKLOADS[name]
        self.w = w
        self.api = api
        self.host = synth.make_attn_inputs(w, seed=seed)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.host.items()}
        self.d = d
        self.max_len = int(self.host["seqlens"].max())
        self.ns = args.num_splits
        self.ws = api.new_attn_workspace(w.B, w.Hq, w.Hkv, w.D, self.max_len, self.ns, dev)
        self.o1 = torch.empty_like(d["q1"])
        self.o2 = torch.empty_like(d["q1"])
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        n_attn = api.decode_attn_num_launches(w.B, w.Hkv, self.max_len, self.ns, w.torch_dtype)
        self.tokens_per_step = w.B
        self.launches_per_step = n_attn + (1 if w.append else 0)
        esize = 4 if w.dtype == "fp32" else 2
        tot = int(self.host["seqlens"].sum())
        self.attn_bytes = attn_algorithmic_bytes(w.B, w.Hq, w.Hkv, w.D, tot, esize)
        self.kv_bytes = tot * w.Hkv * w.D * 2 * esize
        self.units = tot * w.Hkv
        self.bytes_per_unit = w.D * 2 * esize
        self.config = workload_config(name, w, self.host)
        self.path = {"attn_launches": n_attn}
        self.dominant = "dualflow_decode_attn (split kernel, combine inside it)"
        # CUDA graphs: [append] and [attention], replayed every step
        self._append()
        self._attn()
        torch.cuda.synchronize()
        self.g_append = None
        if w.append:
            self.g_append = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_append):
                self._append()
        self.g_attn = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_attn):
            self._attn()
        torch.cuda.synchronize()

    def _append(self):
        d = self.d
        if self.w.append:
            self.api.kv_append(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                               d["block_table"], d["positions"], err_flag=self.err)

    def _attn(self):
        d = self.d
        self.api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], self.max_len, o1=self.o1, o2=self.o2,
                             num_splits=self.ns, workspace=self.ws, err_flag=self.err)

    def step(self, timers=None):
        if self.g_append is not None:
            self.g_append.replay()
        if timers is not None:
            timers["attn"][0].record()
        self.g_attn.replay()
        if timers is not None:
            timers["attn"][1].record()

    def attn_graphs(self):
        """(dual attention graph, primary-only attention graph)."""
        import torch
        d = self.d
        o1 = torch.empty_like(d["q1"])

        def call():
            self.api.decode_attn(d["q1"], None, None, d["k_cache"], d["v_cache"],
                                 d["block_table"], d["seqlens"], self.max_len, o1=o1,
                                 num_splits=self.ns, workspace=self.ws, err_flag=self.err)
        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        self._primary_o1 = o1
        return self.g_attn, g

    def host_io(self):
        import torch
        q = torch.stack([self.host["q1"], self.host["q2raw"]]).pin_memory()
        o = torch.empty_like(q).pin_memory()
        return q, o

    def step_host(self, q_host, o_host):
        d = self.d
        d["q1"].copy_(q_host[0], non_blocking=True)
        d["q2raw"].copy_(q_host[1], non_blocking=True)
        self.step()
        o_host[0].copy_(self.o1, non_blocking=True)
        o_host[1].copy_(self.o2, non_blocking=True)

    def check_err(self):
        return int(self.err.item())


class MixtureRun:
    """Mixture head step: grouped LM-head projection of both flows' final
    hidden states (shared output matrix) + the mixed next-token distribution."""

    timer_keys = ("proj", "mix")
    dominant_key = "proj"

    def __init__(self, args, dev, seed):
        import torch
        from dual_flow_transformer_b200 import api, synth
        w = synth.WORKLOADS["mixture"]
        self.w = w
        self.api = api
        self.host = synth.make_mixture_inputs(w, seed=seed)
        h = self.host
        self.X = torch.cat([h["h1"], h["h2"]]).contiguous().to(dev)
        self.W = h["w_head"].to(dev)
        B, V, d = w.B, w.V, w.d_model
        self.ws = api.new_proj_workspace(2 * B, V, d, "none", dev)
        self.logits = torch.empty((2 * B, V), dtype=torch.bfloat16, device=dev)
        self.p_mix = torch.empty((B, V), dtype=torch.float32, device=dev)
        self.alpha = torch.empty((B,), dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.tokens_per_step = B
        self.launches_per_step = api.grouped_proj_num_launches(2 * B, V, d, "none") + 1
        # LM-head projection: weights once (one [d] row per vocabulary entry),
        # activations in, bf16 logits out
        self.units = V
        self.bytes_per_unit = d * 2
        self.dom_bytes = V * d * 2 + 2 * B * d * 2 + 2 * B * V * 2
        # mixture kernel: logits read once, p_mix and alpha written once
        self.mix_bytes = 2 * B * V * 2 + B * V * 4 + B * 4
        self.config = workload_config("mixture", w, self.host)
        self.path = {}
        self.dominant = "dualflow_grouped_proj (LM head, tcgen05)"
        self._proj()
        self._mix()
        torch.cuda.synchronize()
        self.g_full, self.g_proj, self.g_mix = (torch.cuda.CUDAGraph() for _ in range(3))
        with torch.cuda.graph(self.g_full):
            self._proj()
            self._mix()
        with torch.cuda.graph(self.g_proj):
            self._proj()
        with torch.cuda.graph(self.g_mix):
            self._mix()
        torch.cuda.synchronize()

    def _proj(self):
        self.api.grouped_proj(self.X, self.w.B, self.W, y=self.logits, workspace=self.ws,
                              err_flag=self.err)

    def _mix(self):
        self.api.mixture_head(self.logits, self.w.B, p_mix=self.p_mix, alpha=self.alpha)

    def step(self, timers=None):
        if timers is None:
            self.g_full.replay()
            return
        timers["proj"][0].record()
        self.g_proj.replay()
        timers["proj"][1].record()
        timers["mix"][0].record()
        self.g_mix.replay()
        timers["mix"][1].record()

    def host_io(self):
        import torch
        x = self.X.cpu().pin_memory()
        o = torch.empty(tuple(self.p_mix.shape), dtype=torch.float32).pin_memory()
        return x, o

    def step_host(self, x_host, o_host):
        self.X.copy_(x_host, non_blocking=True)
        self.step()
        o_host.copy_(self.p_mix, non_blocking=True)

    def check_err(self):
        return int(self.err.item())


class MoERun:
    """MoE MLP block of both flows with router replay: route, dispatch, the
    experts' grouped projections, combine (+ residual)."""

    timer_keys = ("experts",)
    dominant_key = "experts"

    def __init__(self, args, dev, seed):
        import torch
        from dual_flow_transformer_b200 import api, synth
        from dual_flow_transformer_b200.moe import DualFlowMoE
        w = synth.WORKLOADS["moe"]
        self.w = w
        self.api = api
        self.host = synth.make_moe_inputs(w, seed=seed)
        h = self.host
        self.x = h["x"].to(dev)
        self.moe = DualFlowMoE(h["w_router"].to(dev), h["w_gu"].to(dev), h["w_down"].to(dev),
                               w.k, w.k_aux, B=w.B, device=dev)
        self.err = self.moe.err
        B, d, F, E = w.B, w.d_model, w.F, w.E
        self.tokens_per_step = B
        self.launches_per_step = self.moe.launches
        self.units = E
        self.bytes_per_unit = 3 * F * d * 2
        rows = 2 * api.MOE_ROWS
        self.dom_bytes = E * (self.bytes_per_unit + rows * d * 2 + rows * F * 2 * 2 + rows * d * 2)
        self.config = workload_config("moe", w, self.host)
        self.path = {}
        self.dominant = "dualflow_grouped_proj (expert SwiGLU projections, tcgen05)"
        self._all()
        torch.cuda.synchronize()
        self.g_full, self.g_pre, self.g_exp, self.g_post = (torch.cuda.CUDAGraph() for _ in range(4))
        with torch.cuda.graph(self.g_full):
            self._all()
        with torch.cuda.graph(self.g_pre):
            self._pre()
        with torch.cuda.graph(self.g_exp):
            self._experts()
        with torch.cuda.graph(self.g_post):
            self._post()
        torch.cuda.synchronize()

    def _pre(self):
        m, w = self.moe, self.w
        self.api.moe_route(self.x, w.B, m.w_router, w.k, w.k_aux, ids=m.ids, g1=m.g1, g2=m.g2)
        self.api.moe_dispatch(self.x, w.B, m.ids, w.E, w.k, w.k_aux, xe=m.xe, slot1=m.slot1,
                              slot2=m.slot2, counts=m.counts, err_flag=m.err)

    def _experts(self):
        self.moe.experts()

    def _post(self):
        m, w = self.moe, self.w
        self.api.moe_combine(m.ye, m.ids, m.g1, m.g2, m.slot1, m.slot2, w.B, w.k, w.k_aux,
                             residual=self.x, y=m.y, err_flag=m.err)

    def _all(self):
        self._pre()
        self._experts()
        self._post()

    def step(self, timers=None):
        if timers is None:
            self.g_full.replay()
            return
        self.g_pre.replay()
        timers["experts"][0].record()
        self.g_exp.replay()
        timers["experts"][1].record()
        self.g_post.replay()

    def host_io(self):
        import torch
        x = self.x.cpu().pin_memory()
        o = torch.empty(tuple(self.moe.y.shape), dtype=torch.bfloat16).pin_memory()
        return x, o

    def step_host(self, x_host, o_host):
        self.x.copy_(x_host, non_blocking=True)
        self.step()
        o_host.copy_(self.moe.y, non_blocking=True)

    def check_err(self):
        return int(self.err.item())


class PrefillRun:
    """Primary prefill of fresh prompts: cache write, causal attention of the
    primary queries, auxiliary query at each last prompt position (one
    dualflow_prefill call = 4 kernels)."""

    timer_keys = ("attn",)
    dominant_key = "attn"
    roof_bound = "tensor"
    metric = PREFILL_METRIC
    profile_prefix = "prefill_attn"
    profile_src = os.path.join(CSRC, "prefill.cu")

    def __init__(self, args, dev, seed):
        import torch
        from dual_flow_transformer_b200 import api, synth
        w = synth.WORKLOADS["prefill"]
        self.w = w
        self.api = api
        self.host = synth.make_prefill_inputs(w, seed=seed)
        h = self.host
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in h.items()}
        self.d = d
        self.ws = api.new_prefill_workspace(h["B"], w.Hq, w.Hkv, w.D, h["max_seqlen"], dev)
        self.o1 = torch.empty_like(d["q1"])
        self.o2 = torch.empty_like(d["q2raw"])
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        lens = (h["cu_seqlens"][1:] - h["cu_seqlens"][:-1]).tolist()
        ctx = h["ctx_lens"].tolist()
        # fresh prompts (no cached prefix) are passed as the API's "no
        # prefix" (ctx_lens = None), as a caller of a fresh prefill would
        self.fresh = all(c == 0 for c in ctx)
        pairs = sum(n * c + n * (n + 1) // 2 for n, c in zip(lens, ctx))
        self.tokens_per_step = h["T"]
        self.launches_per_step = api.prefill_num_launches(True, True)
        self.units = w.Hq * pairs                  # (query row, visible key) pairs, all heads
        self.flops_per_unit = 4 * w.D              # q.k and p*v, multiply-add each
        self.dom_flops = self.units * self.flops_per_unit
        self.config = workload_config("prefill", w, h)
        kern = api.prefill_kernel(w.D, h["T"], self.o1, w.Hq)
        self.dominant = ("dualflow_prefill attention kernel (%s)"
                         % ("tcgen05, TMEM accumulators" if kern == "tcgen05"
                            else "mma.sync, TMA page ring"))
        self.path = {"attn_kernel": kern}
        self._full()
        torch.cuda.synchronize()
        self.g_full, self.g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_full):
            self._full()
        with torch.cuda.graph(self.g_attn):
            self._attn_only()
        torch.cuda.synchronize()

    def _call(self, append, aux):
        d = self.d
        self.api.prefill(d["q1"], d["k_new"] if append else None, d["v_new"] if append else None,
                         d["k_cache"], d["v_cache"], d["block_table"], d["cu_seqlens"],
                         d["max_q_len"], d["max_seqlen"],
                         ctx_lens=None if self.fresh else d["ctx_lens"],
                         q2raw=d["q2raw"] if aux else None, a=d["a"] if aux else None,
                         o1=self.o1, o2=self.o2 if aux else None, workspace=self.ws,
                         err_flag=self.err)

    def _full(self):
        self._call(True, True)

    def _attn_only(self):
        self._call(False, False)   # one launch: the attention kernel alone

    def step(self, timers=None):
        if timers is None:
            self.g_full.replay()
            return
        timers["attn"][0].record()
        self.g_attn.replay()
        timers["attn"][1].record()

    def host_io(self):
        import torch
        h = self.host
        parts = [h["q1"], h["k_new"], h["v_new"], h["q2raw"]]
        n = sum(p.numel() for p in parts)
        x = torch.empty(n, dtype=torch.bfloat16).pin_memory()
        off = 0
        self._views = []
        for p in parts:
            v = x[off:off + p.numel()].view(p.shape)
            v.copy_(p)
            self._views.append(v)
            off += p.numel()
        o = torch.empty(tuple(self.o1.shape), dtype=torch.bfloat16).pin_memory()
        return x, o

    def step_host(self, x_host, o_host):
        d = self.d
        for dst, src in zip((d["q1"], d["k_new"], d["v_new"], d["q2raw"]), self._views):
            dst.copy_(src, non_blocking=True)
        self.step()
        o_host.copy_(self.o1, non_blocking=True)

    def check_err(self):
        return int(self.err.item())


# ----------------------------------------------------------------------------- oracle timing

def _threads_used():
    """Threads the oracle's BLAS uses (its pool size), else the usable cores."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline_record(run, workload, budget_s):
    """The oracle timed on the host: once with the BLAS pool as it stands and
    once limited to one thread (half the budget)."""
    v, sample, el, steps = time_oracle(run, workload, budget_s)
    rec = {"value": v, "unit": "tokens/s", "cores": _threads_used(),
           "usable_cores": len(os.sched_getaffinity(0)), "blas_threads": _threads_used(),
           "kind": "oracle", "sample": sample, "seconds": round(el, 2)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, sample1, el1, _ = time_oracle(run, workload, budget_s / 2)
        rec["one_thread"] = {"value": v1, "unit": "tokens/s", "blas_threads": 1,
                             "sample": sample1, "seconds": round(el1, 2)}
    except Exception as e:  # threadpoolctl missing: say so, do not guess
        rec["one_thread"] = {"value": None, "note": "not measured: %s" % e}
    return rec


def oracle_layer_sample(host, n_seq):
    """Inputs of the oracle for the first n_seq sequences of a layer workload
    (input preparation: dtype widening and page selection, no arithmetic)."""
    import numpy as np
    import torch
    sel = list(range(n_seq))
    tbl = host["block_table"][sel]
    pages = sorted(set(int(p) for p in tbl.flatten().tolist() if p >= 0))
    remap = {p: i for i, p in enumerate(pages)}
    new_tbl = np.array([[remap.get(int(p), -1) for p in row] for row in tbl.tolist()], np.int32)
    f = lambda t: t.to(torch.float32).numpy().astype(np.float64)
    kc = host["k_cache"][pages].to(torch.float32).numpy()
    vc = host["v_cache"][pages].to(torch.float32).numpy()
    return dict(x1=f(host["x1"][sel]), x2=f(host["x2"][sel]), w_qkv=f(host["w_qkv"]),
                w_o=f(host["w_o"]), w_gu=f(host["w_gu"]), w_down=f(host["w_down"]),
                a=f(host["a"]), b=f(host["b"]), c=f(host["c"]), k_cache=kc, v_cache=vc,
                block_table=new_tbl, positions=host["positions"][sel].numpy(),
                Hq=host["Hq"], Hkv=host["Hkv"], D=host["D"], F=host["F"])


def oracle_attn_sample(host, sel):
    import numpy as np
    import torch
    f = lambda t: t.to(torch.float32).numpy()
    return dict(q1=f(host["q1"][sel]), q2raw=f(host["q2raw"][sel]), a=f(host["a"]),
                k_cache=f(host["k_cache"]), v_cache=f(host["v_cache"]),
                block_table=host["block_table"][sel].numpy(),
                seqlens=host["seqlens"][sel].numpy())


def time_oracle(run, workload, budget_s, max_steps=None):
    """Time the oracle on a bounded sample. Returns (tokens/s, sample text,
    seconds, steps). One oracle step = the sample, timed with perf_counter."""
    import oracle
    if workload == "layer":
        n_seq = 1
        inp = oracle_layer_sample(run.host, n_seq)
        t0 = time.perf_counter()
        oracle.layer_step(**inp)
        t1 = time.perf_counter() - t0
        steps = max(1, min(int(budget_s / max(t1, 1e-6)), max_steps or 10 ** 9))
        t0 = time.perf_counter()
        for _ in range(steps):
            oracle.layer_step(**inp)
        el = time.perf_counter() - t0
        sample = ("%d step(s) of the fp64 oracle layer step on %d of %d sequences (both flows), "
                  "full weights, cache %d+1; weights pre-widened to fp64 outside the timing"
                  % (steps, n_seq, run.w.B, run.w.cache_len))
        return n_seq * steps / el, sample, el, steps
    if workload == "mixture":
        return time_oracle_mixture(run.host, budget_s)
    if workload == "moe":
        return time_oracle_moe(run.host, budget_s)
    if workload == "prefill":
        return time_oracle_prefill(run.host, budget_s)
    B = run.w.B
    sel, el, k = [], 0.0, 0
    inp_all = None
    while k < B and el < budget_s:
        sel = [k]
        inp = oracle_attn_sample(run.host, sel)
        t0 = time.perf_counter()
        oracle.decode_attn(**inp)
        el += time.perf_counter() - t0
        k += 1
    sample = "fp64 oracle decode attention (both flows) on %d of %d sequences" % (k, B)
    del inp_all
    return k / el, sample, el, k


def oracle_mixture_sequence(host, b):
    """One sequence of the mixture head on the oracle: fp64 LM-head projection
    of both flows' rows, logits rounded to bf16 (the GPU stores them so), then
    the mixture."""
    import numpy as np
    import oracle
    import torch
    x = torch.stack([host["h1"][b], host["h2"][b]]).to(torch.float32).numpy().astype(np.float64)
    w = host["w_head_f64"]
    logits = oracle.bf16_round(oracle.grouped_proj(x, w, 1))
    return oracle.mixture_head(logits, 1)


def time_oracle_mixture(host, budget_s):
    import numpy as np
    import torch
    if "w_head_f64" not in host:
        host["w_head_f64"] = host["w_head"].to(torch.float32).numpy().astype(np.float64)
    B = host["B"]
    k, el = 0, 0.0
    while el < budget_s and k < 4 * B:
        t0 = time.perf_counter()
        oracle_mixture_sequence(host, k % B)
        el += time.perf_counter() - t0
        k += 1
    sample = ("fp64 oracle mixture head (LM-head projection of both flows + mixture) on %d "
              "sequence(s) of %d; weights pre-widened to fp64 outside the timing" % (k, B))
    return k / el, sample, el, k


def time_oracle_moe(host, budget_s, tokens_per_call=4):
    """The oracle MoE block on a few tokens per call (both flows); the
    experts' weights are widened to fp64 once, outside the timing."""
    import numpy as np
    import oracle
    import torch
    if "w64" not in host:
        f = lambda t: t.to(torch.float32).numpy().astype(np.float64)
        host["w64"] = (f(host["w_router"]), f(host["w_gu"]), f(host["w_down"]))
    wr, wgu, wd = host["w64"]
    x = host["x"].to(torch.float32).numpy().astype(np.float64)
    B = host["B"]
    k, el, calls = 0, 0.0, 0
    while el < budget_s and calls < 64:
        sel = [(k + i) % B for i in range(tokens_per_call)]
        t0 = time.perf_counter()
        oracle.moe_forward(x[sel], x[[B + s for s in sel]], wr, wgu, wd, host["k"], host["k_aux"],
                           x[sel], x[[B + s for s in sel]])
        el += time.perf_counter() - t0
        k += tokens_per_call
        calls += 1
    sample = ("fp64 oracle MoE block (both flows, router replay) on %d token(s) in calls of %d; "
              "expert weights pre-widened to fp64 outside the timing" % (k, tokens_per_call))
    return k / el, sample, el, k


def oracle_prefill_group(host, b, g):
    """Oracle inputs for KV head g of sequence b of a prefill workload: the
    query heads of that group, that head's new K/V and cached pages (input
    selection and dtype widening only, no arithmetic)."""
    import numpy as np
    import torch
    f = lambda t: t.to(torch.float32).numpy()
    Hq, Hkv = host["Hq"], host["Hkv"]
    G = Hq // Hkv
    cu = host["cu_seqlens"].tolist()
    t0, t1 = cu[b], cu[b + 1]
    row = [int(p) for p in host["block_table"][b].tolist() if p >= 0]
    heads = slice(g * G, (g + 1) * G)
    return dict(q1=f(host["q1"][t0:t1, heads]), k_new=f(host["k_new"][t0:t1, g:g + 1]),
                v_new=f(host["v_new"][t0:t1, g:g + 1]),
                k_cache=f(host["k_cache"][row][:, g:g + 1]),
                v_cache=f(host["v_cache"][row][:, g:g + 1]),
                block_table=np.arange(len(row))[None, :], cu_seqlens=np.array([0, t1 - t0]),
                ctx_lens=host["ctx_lens"][b:b + 1].numpy(), q2raw=f(host["q2raw"][b:b + 1, heads]),
                a=f(host["a"][heads]))


def time_oracle_prefill(host, budget_s):
    """The oracle prefill, one (sequence, KV head) group per call: 1/Hkv of
    the work of that sequence's prompt tokens, counted as such."""
    import oracle
    Hkv = host["Hkv"]
    cu = host["cu_seqlens"].tolist()
    el, tokens, calls = 0.0, 0.0, 0
    while el < budget_s and calls < 64:
        b, g = (calls // Hkv) % host["B"], calls % Hkv
        inp = oracle_prefill_group(host, b, g)
        t0 = time.perf_counter()
        oracle.prefill(**inp)
        el += time.perf_counter() - t0
        tokens += (cu[b + 1] - cu[b]) / Hkv
        calls += 1
    sample = ("fp64 oracle prefill (cache write, causal attention, last-position auxiliary "
              "query) on %d (sequence, KV head) group(s) of %d query heads, each counted as 1/%d "
              "of its sequence's prompt tokens" % (calls, host["Hq"] // Hkv, Hkv))
    return tokens / el, sample, el, calls


# ----------------------------------------------------------------------------- main

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from dual_flow_transformer_b200 import synth  # input generators only

    class Host:
        pass

    h = Host()
    if args.workload in ("mixture", "moe", "prefill"):
        h.w = synth.WORKLOADS[args.workload]
        if args.workload == "mixture":
            h.host = synth.make_mixture_inputs(h.w, seed=synth_seed(args.workload))
            v, sample, el, steps = time_oracle_mixture(h.host, 20.0)
        elif args.workload == "prefill":
            h.host = synth.make_prefill_inputs(h.w, seed=synth_seed(args.workload))
            v, sample, el, steps = time_oracle_prefill(h.host, 20.0)
        else:
            h.host = synth.make_moe_inputs(h.w, seed=synth_seed(args.workload))
            v, sample, el, steps = time_oracle_moe(h.host, 20.0)
        line = {"impl": "reference",
                "metric": PREFILL_METRIC if args.workload == "prefill" else METRIC,
                "value": v, "unit": "tokens/s",
                "n_gpus": world, "steps": steps, "steps_requested": args.steps,
                "warmup": args.warmup, "ms_per_step": el / steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_config(args.workload, h.w, h.host, world),
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _threads_used(),
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    if args.workload == "layer":
        h.w = synth.WORKLOADS["layer"]
        h.host = synth.make_layer_inputs(h.w, seed=synth_seed(args.workload))
    else:
        h.w = synth.WORKLOADS[args.workload]
        h.host = synth.make_attn_inputs(h.w, seed=synth_seed(args.workload))
    import oracle
    budget = 150.0
    if args.workload == "layer":
        inp = oracle_layer_sample(h.host, 1)
        t0 = time.perf_counter()
        oracle.layer_step(**inp)
        t1 = time.perf_counter() - t0
        total = args.warmup + args.steps
        steps = args.steps if t1 * total <= budget else max(1, int(budget / t1) - args.warmup)
        warm = min(args.warmup, 1)
        for _ in range(warm):
            oracle.layer_step(**inp)
        t0 = time.perf_counter()
        for _ in range(steps):
            oracle.layer_step(**inp)
        el = time.perf_counter() - t0
        tokens = steps
        sample = ("fp64 oracle layer step on 1 of %d sequences (both flows) per step" % h.w.B)
    else:
        inp = oracle_attn_sample(h.host, [0])
        t0 = time.perf_counter()
        oracle.decode_attn(**inp)
        t1 = time.perf_counter() - t0
        total = args.warmup + args.steps
        steps = args.steps if t1 * total <= budget else max(1, int(budget / t1) - args.warmup)
        t0 = time.perf_counter()
        for i in range(steps):
            oracle.decode_attn(**oracle_attn_sample(h.host, [i % h.w.B]))
        el = time.perf_counter() - t0
        tokens = steps
        sample = "fp64 oracle decode attention on 1 sequence per step"
    value = tokens / el
    cores = _threads_used()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
            "ms_per_step": el / steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.workload, h.w, h.host, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        print("warm-up must be at least 3 steps", file=sys.stderr)
        return 2
    import torch
    world, rank, local = dist_setup(args)
    if world != args.gpus:
        print("--gpus %d but WORLD_SIZE %d" % (args.gpus, world), file=sys.stderr)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    seed_base = synth_seed(args.workload)
    seed = rank_seed(seed_base, rank)
    if args.workload == "layer":
        run = LayerRun(args, dev, seed)
    elif args.workload == "mixture":
        run = MixtureRun(args, dev, seed)
    elif args.workload == "moe":
        run = MoERun(args, dev, seed)
    elif args.workload == "prefill":
        run = PrefillRun(args, dev, seed)
    else:
        run = AttnRun(args, dev, seed, args.workload)

    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()
    if run.check_err():
        print("device error flag %d after warm-up" % run.check_err(), file=sys.stderr)
        return 3

    # ---------------------------------------------------------------- timed region
    keys = getattr(run, "timer_keys", ("attn",))
    timers = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for k in keys} for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    if not args.no_clocks and rank == 0:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark_start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(args.steps):
        run.step()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, world)
    # Second timed pass of the same K steps with events around the attention
    # (the step then runs as separate graphs, so it is not used for `value`).
    torch.cuda.synchronize()
    for i in range(args.steps):
        run.step(timers=timers[i])
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(world)
    clk = clocks.stop() if (not args.no_clocks and rank == 0) else None
    kernel_ms = {k: max_over_ranks(sum(t[k][0].elapsed_time(t[k][1]) for t in timers) / args.steps,
                                   world) for k in keys}
    attn_ms = kernel_ms[getattr(run, "dominant_key", "attn")]

    # ---------------------------------------------------------------- aux overhead
    # Decode attention alone, dual call vs the same call with q2raw = NULL,
    # replayed back to back in A B A B order.
    aux_overhead = None
    if hasattr(run, "attn_graphs"):
        g_dual, g_prim = run.attn_graphs()
        n_rep = max(20, min(args.steps, 400))
        tot = {"dual": 0.0, "primary_only": 0.0}
        for name, g in (("dual", g_dual), ("primary_only", g_prim)) * 2:
            s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(world)
            torch.cuda.synchronize()
            s_ev.record()
            for _ in range(n_rep):
                g.replay()
            e_ev.record()
            torch.cuda.synchronize()
            tot[name] += max_over_ranks(s_ev.elapsed_time(e_ev), world) / (2 * n_rep)
        aux_overhead = {"dual_ms": tot["dual"], "primary_only_ms": tot["primary_only"],
                        "ratio": tot["dual"] / tot["primary_only"], "target": 1.15,
                        "replays": 2 * n_rep,
                        "how": "decode attention graphs alone, dual vs q2raw = NULL, "
                               "ABAB back-to-back replays, CUDA events"}
    err = run.check_err()

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        xh, oh = run.host_io()
        for _ in range(3):
            run.step_host(xh, oh)
        torch.cuda.synchronize()
        barrier(world)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(args.steps):
            run.step_host(xh, oh)
        e2.record()
        torch.cuda.synchronize()
        barrier(world)
        ms2 = max_over_ranks(s2.elapsed_time(e2), world)
        e2e = {"value": world * run.tokens_per_step * args.steps / (ms2 / 1e3),
               "unit": "tokens/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": oh.numel() * oh.element_size()}

    # ---------------------------------------------------------------- CPU baseline (oracle)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_record(run, args.workload, args.cpu_budget_s)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    value = world * run.tokens_per_step * args.steps / (ms_max / 1e3)
    if getattr(run, "roof_bound", "hbm") == "tensor":
        peak, peak_kind = measured_tensor_peak()
        achieved = run.dom_flops / (attn_ms / 1e3) / 1e12
        roofline = {"kernel": run.dominant, "bound": "tensor", "achieved": achieved,
                    "peak": peak, "peak_kind": peak_kind + " (cuBLAS bf16 GEMM, burst, "
                    "MEASURED_PEAKS.json)" if peak_kind == "measured" else peak_kind,
                    "unit": "TFLOP/s", "frac": achieved / peak,
                    "traffic": traffic_from_profile(args.workload, run.profile_prefix,
                                                    run.profile_src),
                    "algorithmic_flops_per_launch": run.dom_flops,
                    "units_per_launch": run.units, "flops_per_unit": run.flops_per_unit}
        peak, peak_kind = measured_hbm_peak()
    else:
        peak, peak_kind = measured_hbm_peak()
        dom_bytes = getattr(run, "dom_bytes", None) or run.attn_bytes
        achieved = dom_bytes / (attn_ms / 1e3) / 1e9
        roofline = {"kernel": run.dominant, "bound": "hbm", "achieved": achieved,
                    "peak": peak, "peak_kind": peak_kind + " (STREAM-style copy, "
                    "MEASURED_PEAKS.json)" if peak_kind == "measured" else peak_kind,
                    "unit": "GB/s", "frac": achieved / peak,
                    "traffic": traffic_from_profile(args.workload),
                    "algorithmic_bytes_per_launch": dom_bytes,
                    "units_per_launch": run.units, "bytes_per_unit": run.bytes_per_unit}
    line = {
        "metric": getattr(run, "metric", METRIC), "value": value, "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations/cache, N(0,0.02) weights, N(0,0.1) couplings)",
        "config": dict(run.config, parallelism="replicas" if world > 1 else "single GPU"),
        "path": run.path,
        "dominant_ms_per_launch": attn_ms,
        "kernel_timing": "second pass of the same %d steps, the timed kernels' graphs bracketed "
                         "by CUDA events on the launching stream (value uses the single-graph "
                         "step)" % args.steps,
        "roofline": roofline,
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": run.launches_per_step * args.steps,
        "clocks": clk, "device_error_flag": err,
    }
    if aux_overhead is not None:
        line["aux_overhead"] = aux_overhead
    if hasattr(run, "kv_bytes"):
        line["kv_read_gbs"] = run.kv_bytes / (attn_ms / 1e3) / 1e9
        line["kv_frac_of_hbm_peak"] = run.kv_bytes / (attn_ms / 1e3) / 1e9 / peak
        line["kv_frac_of_nominal_8tbs"] = run.kv_bytes / (attn_ms / 1e3) / 1e9 / NOMINAL_HBM_GBS
    if hasattr(run, "mix_bytes"):
        mix_gbs = run.mix_bytes / (kernel_ms["mix"] / 1e3) / 1e9
        line["mixture_kernel"] = {"kernel": "dualflow_mixture_head", "bound": "hbm",
                                  "ms_per_launch": kernel_ms["mix"], "achieved": mix_gbs,
                                  "peak": peak, "unit": "GB/s", "frac": mix_gbs / peak,
                                  "algorithmic_bytes_per_launch": run.mix_bytes}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def synth_seed(workload):
    from dual_flow_transformer_b200 import synth
    return synth.WORKLOADS[workload].seed


if __name__ == "__main__":
    sys.exit(main())
