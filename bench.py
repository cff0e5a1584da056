#!/usr/bin/env python
"""Benchmark: K8/V4 quantised-KV decode attention on B200.

One step = one decode step of the workload over all its attention layers:
per layer, the quantise-and-append of the step's new tokens (when the workload
appends) followed by split-K decode attention and the LSE combine, all through
the C ABI.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--kv-format k8v4|k8v8|f8|k4v4|bf16] [--impl ours|reference]
                  [--sharded] [--replicas]

At N > 1 (one process per GPU under torchrun) the step is the decode of one
request split by context over the ranks (strong scaling: every rank decodes
its own keys, one NCCL all-gather of packed partials and a merge per layer);
--replicas runs N independent copies of the request instead.

--workload prefill_chunk measures chunked-prefill attention instead: per layer
the 1024-token chunk's append and nf_prefill_attn, reported as chunk tokens/s
and the prefill kernel's TFLOP/s against the measured tensor-core peak.

Metric: KV tokens/s (each cached key counted once per layer, heads not
multiplied) and the decode kernel's achieved HBM GB/s against the measured B200
copy bandwidth.  Inputs are seeded synthetic tensors of the workload's shape,
resident in HBM before timing; the KV bytes of one step exceed the 126 MB L2,
so successive steps stream from HBM.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "KV tokens/s and achieved HBM GB/s (% of B200 peak) for K8/V4 decode attn"
UNIT = "KV tokens/s"
DEFAULT_WORKLOAD = "longest"
# The other workloads of >= 64K keys: at N = 1 their decode roofline and step
# time are measured after the headline and reported beside it (key "others").
OTHER_WORKLOADS = ["ragged_c2", "mtp_verify"]
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ["long_context_quantized_b200/csrc/nf_decode.cuh",
                  "long_context_quantized_b200/csrc/nf_decode_tc.cuh",
                  "long_context_quantized_b200/csrc/nf_tc.cuh",
                  "long_context_quantized_b200/csrc/nf_common.cuh",
                  "long_context_quantized_b200/csrc/nf_api.cu"]


# ------------------------------------------------------------------ helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for s in DECODE_SOURCES:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, fmt):
    """dram bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{fmt}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(x, device=None):
    """The largest of the ranks' values of x (every rank gets it); x itself
    when no process group is up.  Timings of the weak-scaled replicas are
    reduced with it, so the job's time is that of its slowest rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world_size, ms_max):
    """Whole-job KV tokens/s: every rank processes its own replica of the
    workload, so the job's tokens are world_size times a rank's, over the
    slowest rank's time."""
    return tokens_per_rank * world_size / (ms_max / 1e3)


# ------------------------------------------------------------ GPU workload
class GpuWorkload:
    """All layers' pools, queries and step inputs resident on the device."""

    def __init__(self, w, fmt_name, device):
        import long_context_quantized_b200 as nf
        self.nf = nf
        self.w = w
        self.dev = device
        self.fmt_name = fmt_name
        self.fmt = {"k8v4": nf.NF_KV_K8V4, "k8v8": nf.NF_KV_K8V8, "f8": nf.NF_KV_F8, "k4v4": nf.NF_KV_K4V4,
                    "bf16": nf.NF_KV_BF16}[fmt_name]
        self.decode_flags = nf.NF_DECODE_EARLY_KV
        assert w.n_new in (0, w.n_q), "the early-KV guarantee needs n_new == n_q"
        bt = workloads.block_table(w)
        self.bt = torch.as_tensor(bt, dtype=torch.int32, device=device)
        self.seqlens = torch.as_tensor(w.seqlens, dtype=torch.int32, device=device)
        self.before = torch.as_tensor(w.cached, dtype=torch.int32, device=device)
        self.max_seqlen = max(w.seqlens)
        self.layers, self.q, self.knew, self.vnew, self.out = [], [], [], [], []
        for layer in range(w.layers):
            kv = nf.KVLayer.empty(self.fmt, w.pool_blocks, w.num_kv_heads, device=device, fill=0)
            knew, vnew = [], []
            for b in range(w.batch):
                k, v = workloads.layer_kv(w, layer, b, device=device)
                c = w.cached[b]
                nf.nf_kv_append_quant(kv, k[None, :c].contiguous(), v[None, :c].contiguous(), self.bt[b:b + 1],
                                      torch.zeros(1, dtype=torch.int32, device=device))
                knew.append(k[c:])
                vnew.append(v[c:])
                del k, v
            self.layers.append(kv)
            if w.n_new:
                self.knew.append(torch.stack(knew).contiguous())
                self.vnew.append(torch.stack(vnew).contiguous())
            self.q.append(workloads.layer_q(w, layer, device=device))
        # every layer's inputs and outputs live in one tensor per kind (the layers'
        # tensors are views), so a step's host copies are one transfer each
        self.q_all = torch.stack(self.q).contiguous()
        self.q = [self.q_all[i] for i in range(w.layers)]
        if w.n_new:
            self.knew_all = torch.stack(self.knew).contiguous()
            self.vnew_all = torch.stack(self.vnew).contiguous()
            self.knew = [self.knew_all[i] for i in range(w.layers)]
            self.vnew = [self.vnew_all[i] for i in range(w.layers)]
        self.out_all = torch.empty((w.layers, w.batch, w.n_q, w.num_q_heads, 128), dtype=torch.float32, device=device)
        self.out = [self.out_all[i] for i in range(w.layers)]
        ws = nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, self.max_seqlen)
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=device)
        torch.cuda.synchronize()
        assert nf.nf_get_device_error() == 0

    def append(self, layer):
        if self.w.n_new:
            self.nf.nf_kv_append_quant(self.layers[layer], self.knew[layer], self.vnew[layer], self.bt, self.before)

    def decode(self, layer):
        # the step appends (when it appends) exactly the n_q newest tokens right
        # before each decode, and lengths and tables stay fixed: the early-KV
        # guarantee of nf_decode_attn_ex holds
        w = self.w
        self.nf.nf_decode_attn_ex(self.layers[layer], self.q[layer], self.bt, self.seqlens, self.max_seqlen,
                                  w.softmax_scale, w.causal, self.decode_flags, self.out[layer], None, self.ws)

    def step(self):
        for layer in range(self.w.layers):
            self.append(layer)
            self.decode(layer)

    # --- byte accounting (algorithmic, per decode launch / per step)
    def kv_bytes_per_layer(self):
        per = workloads.kv_bytes_per_token_head(self.fmt_name)
        return sum(self.w.seqlens) * self.w.num_kv_heads * per

    def decode_bytes_per_launch(self):
        w = self.w
        q = self.q[0].numel() * self.q[0].element_size()
        out = w.batch * w.n_q * w.num_q_heads * 128 * 4
        tables = sum(math.ceil(L / 256) for L in w.seqlens) * 4 + 4 * w.batch
        return self.kv_bytes_per_layer() + q + out + tables

    def step_bytes(self):
        w = self.w
        per = workloads.kv_bytes_per_token_head(self.fmt_name)
        app = w.batch * w.n_new * w.num_kv_heads * (per + 2 * 128 * 2)
        return w.layers * (self.decode_bytes_per_launch() + app)

    def launches_per_step(self):
        # per layer: the append kernel (when the step appends) and the decode
        # kernel, whose cross-CTA combine is fused in
        return self.w.layers * ((1 if self.w.n_new else 0) + 1)


def time_graph(g, steps, warmup, stream):
    """Mean ms per replay: events and replays on the same stream."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def time_decode_stream(gw, steps, stream):
    """Average duration of one nf_decode_attn launch when the step's decode
    launches run back to back (as they do inside the step: each may start while
    the previous one finishes): CUDA events around replays of a graph holding
    the decode call of every layer, divided by the number of launches."""
    L = gw.w.layers
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for layer in range(L):
            gw.decode(layer)
    ms = time_graph(g, steps, 3, stream)
    del g
    return ms / L


def time_decode_launches(gw, steps, stream):
    """Average duration of one nf_decode_attn call (one fused kernel launch)
    timed in isolation: CUDA events recorded around every call inside a
    captured graph (the events keep consecutive launches from overlapping)."""
    L = gw.w.layers
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(L)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for layer in range(L):
            ev[layer][0].record()
            gw.decode(layer)
            ev[layer][1].record()
    tot, n = 0.0, 0
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        for _ in range(steps):
            g.replay()
            torch.cuda.synchronize()
            for a, b in ev:
                tot += a.elapsed_time(b)
                n += 1
    return tot / n


def measure_e2e(gw, args, stream, device):
    """End to end: the step's inputs (every layer's q and new K/V) copied from
    pinned host memory, the step, every layer's output copied back; returns
    (ms per step, max over ranks; H2D bytes; D2H bytes)."""
    h_in = [gw.q_all.cpu().pin_memory()]
    d_in = [gw.q_all]
    if gw.w.n_new:
        h_in += [gw.knew_all.cpu().pin_memory(), gw.vnew_all.cpu().pin_memory()]
        d_in += [gw.knew_all, gw.vnew_all]
    h_out = torch.empty_like(gw.out_all, device="cpu").pin_memory()
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        for d, hsrc in zip(d_in, h_in):
            d.copy_(hsrc, non_blocking=True)
        gw.step()
        h_out.copy_(gw.out_all, non_blocking=True)
    e2e_ms = time_graph(ge, args.steps, max(3, args.warmup), stream)
    e2e_ms = max_over_ranks(e2e_ms, device)
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out.numel() * h_out.element_size()
    del ge
    torch.cuda.synchronize()
    return e2e_ms, h2d, d2h


# ------------------------------------------------ context-sharded decode leg
class ShardedWorkload:
    """One rank's shard of the workload (long_context_quantized_b200.sharded):
    a pool holding only this rank's blocks of every layer, the replicated
    queries, and one ShardedDecoder (its packed slot, gather buffer and
    workspace reused by every layer).  The step's appended tokens belong to
    the last shard (every shard boundary lies at or before L - n_q), so only
    the last rank appends."""

    def __init__(self, w, fmt_name, device, world, rank, group=None):
        import long_context_quantized_b200 as nf
        from long_context_quantized_b200 import sharded
        self.nf, self.w, self.dev = nf, w, device
        self.fmt_name = fmt_name
        fmt = {"k8v4": nf.NF_KV_K8V4, "k8v8": nf.NF_KV_K8V8, "f8": nf.NF_KV_F8, "k4v4": nf.NF_KV_K4V4,
               "bf16": nf.NF_KV_BF16}[fmt_name]
        self.spec = sharded.shard_plan(list(w.seqlens), w.n_q, world, w.causal)[rank]
        self.local_bt = sharded.local_pool_table(self.spec, device)
        n_local = max(1, sum(self.spec.n_blocks))
        self.layers, self.q, self.knew, self.vnew = [], [], [], []
        new_before = []  # local position of the first new token, per sequence (this rank holds them)
        for b in range(w.batch):
            pos = sharded.shard_positions(self.spec, b)
            new_before.append(w.cached[b] - pos.start if (w.n_new and pos.stop > w.cached[b]) else None)
        self.appends = w.n_new > 0 and all(x is not None for x in new_before)
        self.before = torch.as_tensor([x or 0 for x in new_before], dtype=torch.int32, device=device)
        for layer in range(w.layers):
            kv = nf.KVLayer.empty(fmt, n_local, w.num_kv_heads, device=device, fill=0)
            kn, vn = [], []
            for b in range(w.batch):
                pos = sharded.shard_positions(self.spec, b)
                if not len(pos):
                    continue
                k, v = workloads.layer_kv(w, layer, b, device=device)
                end = min(pos.stop, w.cached[b])
                if end > pos.start:
                    nf.nf_kv_append_quant(kv, k[None, pos.start:end].contiguous(), v[None, pos.start:end].contiguous(),
                                          self.local_bt[b:b + 1], torch.zeros(1, dtype=torch.int32, device=device))
                if self.appends:
                    kn.append(k[w.cached[b]:pos.stop])
                    vn.append(v[w.cached[b]:pos.stop])
                del k, v
            self.layers.append(kv)
            if self.appends:
                self.knew.append(torch.stack(kn).contiguous())
                self.vnew.append(torch.stack(vn).contiguous())
            self.q.append(workloads.layer_q(w, layer, device=device))
        self.dec = sharded.ShardedDecoder(self.spec, w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, device, group)
        self.out_all = torch.empty((w.layers, w.batch, w.n_q, w.num_q_heads, 128), dtype=torch.float32, device=device)
        self.lse_all = torch.empty((w.layers, w.batch, w.n_q, w.num_q_heads), dtype=torch.float32, device=device)
        torch.cuda.synchronize()
        assert nf.nf_get_device_error() == 0

    def layer(self, i):
        if self.appends:
            self.nf.nf_kv_append_quant(self.layers[i], self.knew[i], self.vnew[i], self.local_bt, self.before)
        self.dec(self.layers[i], self.q[i], self.local_bt, self.w.softmax_scale, self.out_all[i], self.lse_all[i])

    def step(self):
        for i in range(self.w.layers):
            self.layer(i)

    def local_decode_bytes(self):
        per = workloads.kv_bytes_per_token_head(self.fmt_name)
        return sum(self.spec.lengths) * self.w.num_kv_heads * per


def sharded_main(args, w, ws, rank, local):
    """The decode step of one request split by context over the ranks: every
    rank decodes its own keys, the ranks exchange one packed partial per
    layer (NCCL all-gather) and merge it.  Total work is fixed as N grows
    (strong scaling); the step is timed eagerly (no CUDA graph around the
    collectives) with CUDA events, max over ranks."""
    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    group = None
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    sw = ShardedWorkload(w, args.kv_format, device, ws, rank, group)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(3, args.warmup)):
        sw.step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        sw.step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    if ws > 1:
        dist.barrier()
    err = sw.nf.nf_get_device_error()
    assert err == 0, f"device error {err}"
    tokens = w.kv_tokens_per_step()  # the whole request: every key once per layer, over all ranks
    value = tokens / (ms / 1e3)
    # this rank's decode launch alone (no exchange), back to back: the roofline
    g = torch.cuda.CUDAGraph()
    gs = torch.cuda.Stream(device=device)
    from long_context_quantized_b200 import sharded
    with torch.cuda.graph(g, stream=gs):
        for i in range(w.layers):
            sharded.decode_partial_into(sw.layers[i], sw.q[i], sw.spec, sw.local_bt, w.softmax_scale, sw.dec.slot,
                                        sw.dec.workspace, sw.dec.seqlens)
    dec_ms = time_graph(g, max(5, min(args.steps, 30)), 3, gs) / w.layers
    del g
    dec_ms = max_over_ranks(dec_ms, device)
    peak, peak_kind = measured_peaks()
    dec_bytes = sw.local_decode_bytes()
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    # end to end: every layer's q from pinned host memory, every layer's output back
    h_q = [t.cpu().pin_memory() for t in sw.q]
    h_out = torch.empty_like(sw.out_all, device="cpu").pin_memory()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(args.steps):
        for i in range(w.layers):
            sw.q[i].copy_(h_q[i], non_blocking=True)
            sw.layer(i)
        h_out.copy_(sw.out_all, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": DTYPES[args.kv_format], "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlens": list(w.seqlens), "n_q": w.n_q,
                   "n_new": w.n_new, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads, "layers": w.layers,
                   "kv_format": args.kv_format, "causal": w.causal,
                   "parallelism": f"context split over {ws} GPU(s): per layer the local decode, one NCCL "
                                  "all-gather of packed (o, lse) partials, nf_attn_combine_packed",
                   "l2": "KV bytes per step %.1f MB > 126 MB L2" % (sw.local_decode_bytes() * ws * w.layers / 1e6),
                   "timing": "eager step (no CUDA graph around the collectives), CUDA events, max over ranks"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "decode_kernel of one rank's shard (back to back, no exchange)",
                     "peak_source": peak_kind, "bytes_per_launch": dec_bytes, "launch_us": dec_ms * 1e3},
        "cpu_baseline": None,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_q),
                "d2h_bytes_per_step": h_out.numel() * h_out.element_size()},
        "gpu_launches": (w.layers * ((1 if sw.appends else 0) + 1 + (1 if ws > 1 else 0))) * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- chunked prefill leg
PREFILL_METRIC = "prefill chunk tokens/s through chunked-prefill attention over the K8/V4 cache (all layers)"
PREFILL_UNIT = "tokens/s"


class PrefillWorkload(GpuWorkload):
    """The last chunk of a prompt: per layer the chunk's K/V appended, then
    nf_prefill_attn of its n_q queries against the whole cache."""

    def decode(self, layer):
        w = self.w
        self.nf.nf_prefill_attn(self.layers[layer], self.q[layer], self.bt, self.seqlens, self.max_seqlen,
                                w.softmax_scale, w.causal, self.out[layer], None)

    def flops_per_launch(self):
        """2 x 2 x d per (query row, visible key): S = Q . K^T and O = P . V."""
        w = self.w
        keys = 0
        for L in w.seqlens:
            if w.causal:
                keys += sum(L - w.n_q + j + 1 for j in range(w.n_q))
            else:
                keys += L * w.n_q
        return 4 * w.head_dim * w.num_q_heads * keys


def prefill_oracle_sample(w, budget_s=12.0, device="cpu"):
    """Time the oracle on rows of the chunk (layer 0, kv-head 0, positions
    spread over the chunk, all G heads), about budget_s seconds.  Returns
    (chunk tokens/s for the whole step, threads, description, s per rep)."""
    import oracle
    bt = workloads.block_table(w)
    pool = oracle.Pool(oracle.FMT_K8V4, w.pool_blocks, 1, 128, poison=0)
    for b in range(w.batch):
        k, v = workloads.layer_kv(w, 0, b, device=device)
        oracle.append(pool, k[:, :1].float().cpu().numpy()[None], v[:, :1].float().cpu().numpy()[None],
                      bt[b:b + 1], np.zeros(1, np.int32))
        del k, v
    q = workloads.layer_q(w, 0, device=device)[:, :, :w.group].float().cpu().numpy()
    threads = os.cpu_count() or 1
    sl = np.array(w.seqlens, np.int32)
    pos = np.linspace(0, w.n_q - 1, max(1, min(w.n_q, 2 * threads))).round().astype(np.int64)
    rows = np.array([j * w.group + gh for j in pos for gh in range(w.group)], np.int64)
    reps, t_tot = 0, 0.0
    while True:
        t0 = time.perf_counter()
        oracle.decode_attn(pool, q, bt, sl, w.softmax_scale, w.causal, rows=rows, nthreads=threads)
        t_tot += time.perf_counter() - t0
        reps += 1
        if t_tot >= budget_s or reps >= 50:
            break
    rows_per_s = len(rows) * reps / t_tot
    value = rows_per_s / (w.num_q_heads * w.layers)  # a chunk token is H_q rows in each layer
    desc = (f"oracle (C, fp64 attention) on {threads} host threads: {len(rows)} query rows (positions "
            f"spread over the {w.n_q}-token chunk, all {w.group} heads of kv-head 0, layer 0), {reps} "
            f"repetition(s), {t_tot:.1f} s; tokens = rows / (H_q x layers)")
    return value, threads, desc, t_tot / reps


def prefill_main(args, w, ws, rank, local):
    import long_context_quantized_b200 as nf
    if args.impl == "reference":
        if rank != 0:
            return
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        value, threads, desc, _ = prefill_oracle_sample(w, budget_s=min(12.0, 3.0 * max(1, args.steps)),
                                                        device=dev)
        line = {"metric": PREFILL_METRIC, "value": value, "unit": PREFILL_UNIT, "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.n_q * w.batch / value * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": w.name, "kv_format": "k8v4", "step": "oracle sample"},
                "cpu_baseline": {"value": value, "unit": PREFILL_UNIT, "cores": threads, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": PREFILL_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    gw = PrefillWorkload(w, "k8v4", device)
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        gw.step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        gw.step()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = time_graph(g, args.steps, 0, stream)
    clk = clocks.stop()
    ms = max_over_ranks(ms, device)
    if ws > 1:
        torch.distributed.barrier()
    err = nf.nf_get_device_error()
    assert err == 0, f"device error {err}"
    tokens = w.n_q * w.batch
    value = job_throughput(tokens, ws, ms)

    pf_ms = time_decode_stream(gw, max(3, min(args.steps, 10)), stream)
    pf_iso_ms = time_decode_launches(gw, max(3, min(args.steps, 10)), stream)
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) if os.path.exists(
            os.path.join(ROOT, "MEASURED_PEAKS.json")) else open(os.devnull) as f:
        txt = f.read()
    peaks = json.loads(txt) if txt else {}
    # fp16 and bf16 run at the same tensor-core rate; the launches run back to
    # back for seconds, so the sustained figure applies
    peak = float(peaks.get("bf16_tflops_sustained", 1400.0))
    peak_kind = "measured bf16 sustained (fp16 at the same rate)" if peaks else "fallback"
    flops = gw.flops_per_launch()
    achieved = flops / (pf_ms / 1e3) / 1e12

    e2e_ms, h2d, d2h = measure_e2e(gw, args, stream, device)
    del g
    torch.cuda.synchronize()
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cv, threads, desc, _ = prefill_oracle_sample(w, budget_s=12.0, device=device)
        cpu = {"value": cv, "unit": PREFILL_UNIT, "cores": threads, "kind": "oracle", "sample": desc}
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": PREFILL_METRIC, "value": value, "unit": PREFILL_UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8/s4 KV codes dequantised to f16, tcgen05 f16 tensor-core products, f32 softmax/accumulate",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlens": list(w.seqlens), "n_q": w.n_q,
                   "n_new": w.n_new, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
                   "layers": w.layers, "kv_format": "k8v4", "causal": w.causal,
                   "l2": "KV bytes per step %.0f MB > 126 MB L2" % (gw.kv_bytes_per_layer() * w.layers / 1e6),
                   "timing": "CUDA graph of one step, CUDA events, max over ranks"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "prefill_kernel (nf_prefill_attn)", "peak_source": peak_kind,
                     "flops_per_launch": flops, "launch_us": pf_ms * 1e3, "launch_us_isolated": pf_iso_ms * 1e3},
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(tokens, ws, e2e_ms), "unit": PREFILL_UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": gw.launches_per_step() * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ CPU oracle leg
def oracle_sample(w, fmt_name, budget_s=12.0, device="cpu"):
    """Time the CPU oracle on a bounded sample of the workload: decode attention
    of the rows of kv-head 0 of layer 0 (G * n_q rows per sequence), repeated
    until about budget_s seconds.  Returns (KV tokens/s, threads, description).
    KV tokens counts each key once per kv-head processed, scaled by 1 / H_kv."""
    import oracle
    fmt = {"k8v4": oracle.FMT_K8V4, "k8v8": oracle.FMT_K8V8, "f8": oracle.FMT_F8, "k4v4": oracle.FMT_K4V4,
           "bf16": oracle.FMT_BF16}[fmt_name]
    bt = workloads.block_table(w)
    pool = oracle.Pool(fmt, w.pool_blocks, 1, 128, poison=0)
    for b in range(w.batch):
        k, v = workloads.layer_kv(w, 0, b, device=device)
        oracle.append(pool, k[:, :1].float().cpu().numpy()[None], v[:, :1].float().cpu().numpy()[None],
                      bt[b:b + 1], np.zeros(1, np.int32))
        del k, v
    q = workloads.layer_q(w, 0, device=device)[:, :, :w.group].float().cpu().numpy()
    threads = os.cpu_count() or 1
    sl = np.array(w.seqlens, np.int32)
    reps, t_tot = 0, 0.0
    while True:
        t0 = time.perf_counter()
        oracle.decode_attn(pool, q, bt, sl, w.softmax_scale, w.causal, nthreads=threads)
        t_tot += time.perf_counter() - t0
        reps += 1
        if t_tot >= budget_s or reps >= 50:
            break
    tokens = sum(w.seqlens) * reps / w.num_kv_heads
    desc = (f"oracle (C, fp64 attention) on {threads} host threads: layer 0, kv-head 0 of "
            f"{w.num_kv_heads} ({w.group * w.n_q} query rows per sequence), {reps} repetition(s), "
            f"{t_tot:.1f} s; KV tokens scaled by 1/{w.num_kv_heads}")
    return tokens / t_tot, threads, desc, t_tot / reps


# --------------------------------------------------------------------- main
DTYPES = {
    "k8v4": "s8/s4 KV codes, f16 tensor-core products, f32 softmax/accumulate",
    "k8v8": "s8/s8 KV codes, f16 tensor-core products, f32 softmax/accumulate",
    "f8": "e4m3 KV codes, f16 tensor-core products, f32 softmax/accumulate",
    "k4v4": "s4/s4 KV codes with power-of-two scales, s8 and f16 tensor-core products, f32 softmax/accumulate",
    "bf16": "bf16 KV, bf16 tensor-core products, f32 softmax/accumulate",
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=workloads.ORDER + list(workloads.PREFILL))
    ap.add_argument("--kv-format", default="k8v4", choices=["k8v4", "k8v8", "f8", "k4v4", "bf16"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the other >= 64K workloads measured after the headline at N = 1")
    ap.add_argument("--sharded", action="store_true",
                    help="at N = 1: the context-sharded path (the default at N > 1)")
    ap.add_argument("--replicas", action="store_true",
                    help="at N > 1: independent replicas of the whole request instead of the context split")
    ap.add_argument("--layers", type=int, default=None,
                    help="profiling only: run fewer layers than the workload has")
    args = ap.parse_args()
    ws, rank, local = dist_env()
    w = workloads.get(args.workload)
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layers=args.layers)

    if w.name in workloads.PREFILL:
        return prefill_main(args, w, ws, rank, local)

    if args.impl == "reference":
        if rank != 0:
            return
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        per_step = []
        value, threads, desc, t_rep = oracle_sample(w, args.kv_format, budget_s=0.0, device=dev)
        for _ in range(args.warmup):
            oracle_sample(w, args.kv_format, budget_s=0.0, device=dev)
        for _ in range(args.steps):
            v, threads, desc, t_rep = oracle_sample(w, args.kv_format, budget_s=0.0, device=dev)
            per_step.append(t_rep)
        t = sum(per_step) / len(per_step)
        value = sum(w.seqlens) / w.num_kv_heads / t
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": {"workload": w.name, "kv_format": args.kv_format, "step": "oracle sample"},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if (ws > 1 and not args.replicas) or args.sharded:
        return sharded_main(args, w, ws, rank, local)

    import long_context_quantized_b200 as nf
    if ws > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    gw = GpuWorkload(w, args.kv_format, device)
    stream = torch.cuda.Stream(device=device)

    # ---- the step as a CUDA graph
    with torch.cuda.stream(stream):
        gw.step()   # eager warm-up, outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        gw.step()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = time_graph(g, args.steps, 0, stream)
    clk = clocks.stop()
    ms = max_over_ranks(ms, device)
    if ws > 1:
        torch.distributed.barrier()
    err = nf.nf_get_device_error()
    assert err == 0, f"device error {err}"

    tokens = w.kv_tokens_per_step()
    value = job_throughput(tokens, ws, ms)

    # ---- dominant kernel: per-launch duration, back to back and in isolation
    dec_ms = time_decode_stream(gw, max(5, min(args.steps, 30)), stream)
    dec_iso_ms = time_decode_launches(gw, max(5, min(args.steps, 30)), stream)
    peak, peak_kind = measured_peaks()
    dec_bytes = gw.decode_bytes_per_launch()
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    traffic = recorded_traffic(w.name, args.kv_format)

    e2e_ms, h2d, d2h = measure_e2e(gw, args, stream, device)
    del g
    torch.cuda.synchronize()

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cv, threads, desc, _ = oracle_sample(w, args.kv_format, budget_s=12.0, device=device)
        cpu = {"value": cv, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    launches = gw.launches_per_step() * args.steps
    kv_step_bytes = gw.kv_bytes_per_layer() * w.layers
    step_bytes = gw.step_bytes()
    others = None
    if ws == 1 and w.name == DEFAULT_WORKLOAD and not args.no_others and not args.layers:
        del gw
        torch.cuda.empty_cache()
        others = {name: measure_other(workloads.get(name), args, device) for name in OTHER_WORKLOADS}

    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    l2_note = ("KV bytes per step %.1f MB > 126 MB L2: no flush needed" % (kv_step_bytes / 1e6)
               if kv_step_bytes > 126e6 else "L2-resident (correctness-size workload)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPES[args.kv_format],
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlens": list(w.seqlens), "n_q": w.n_q,
                   "n_new": w.n_new, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
                   "layers": w.layers, "kv_format": args.kv_format, "causal": w.causal,
                   "l2": l2_note, "timing": "CUDA graph of one step, CUDA events, max over ranks",
                   "decode_flags": "NF_DECODE_EARLY_KV"},
        "step_gbs": step_bytes / (ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "decode_kernel (nf_decode_attn: split-K with fused combine)", "peak_source": peak_kind,
                     "bytes_per_launch": dec_bytes, "launch_us": dec_ms * 1e3,
                     "launch_us_isolated": dec_iso_ms * 1e3,
                     "frac_isolated": dec_bytes / (dec_iso_ms / 1e3) / 1e9 / peak},
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(tokens, ws, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if others is not None:
        line["others"] = others
    print(json.dumps(line), flush=True)


def measure_other(w, args, device):
    """The decode step of another workload, measured like the headline (step
    graph timed with CUDA events, decode launches back to back for the
    roofline), for the line's "others" key.  Returns a dict."""
    steps = max(5, min(args.steps, 30))
    gw = GpuWorkload(w, args.kv_format, device)
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        gw.step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        gw.step()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    time.sleep(0.3)
    ms = time_graph(g, steps, 0, stream)
    dec_ms = time_decode_stream(gw, steps, stream)
    clk = clocks.stop()
    err = gw.nf.nf_get_device_error()
    assert err == 0, f"device error {err}"
    peak, peak_kind = measured_peaks()
    dec_bytes = gw.decode_bytes_per_launch()
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    res = {
        "metric": METRIC, "value": w.kv_tokens_per_step() / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
        "steps": steps, "step_gbs": gw.step_bytes() / (ms / 1e3) / 1e9,
        "config": {"workload": w.name, "batch": w.batch, "seqlens": list(w.seqlens), "n_q": w.n_q,
                   "n_new": w.n_new, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads, "layers": w.layers,
                   "kv_format": args.kv_format, "causal": w.causal},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(w.name, args.kv_format), "peak_source": peak_kind,
                     "bytes_per_launch": dec_bytes, "launch_us": dec_ms * 1e3},
        # the timed step graph and the timed graph of back-to-back decode launches
        "gpu_launches": gw.launches_per_step() * steps + w.layers * steps,
        "clocks": clk,
    }
    del g, gw
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


if __name__ == "__main__":
    main()
