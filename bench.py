#!/usr/bin/env python
"""Benchmark of the QSA layer on B200 (one process per GPU).

Default workload: QSA prefill of one 1M-token sequence (16 query heads, 2 KV
heads, head dim 128, indexer 4 x 64, r = 4, token budget 2048) -- the context
length the pages quote their attention speed-up at.  One step = the whole hot
path: qsa_pool -> qsa_index_topk -> qsa_sparse_attn_prefill on inputs already
in HBM.  With N GPUs every rank runs its own independent sequence (weak
scaling, no data-path collective); the time is the max over ranks.

The JSON line also carries: the dominant kernel's roofline fraction (CUDA
events on the launch stream), an end-to-end figure through the C ABI with
host buffers (H2D copies of the inputs and D2H of the output inside the timed
region), the CPU oracle timed on a bounded sample of the same workload, the
library's dense GQA attention on the same inputs (speed-up context), and
secondary measurements (128K prefill, 64 x 256K decode).

``--impl reference`` times the CPU oracle instead (the reference arm).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_long_10_b200 import synth  # noqa: E402

METRIC = "QSA layer prefill tokens/s at 128K/1M; decode us/token at 256K; % roofline"
L2_BYTES = 126 * 2**20
BF = torch.bfloat16


# ----------------------------------------------------------------- helpers --

def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            sel = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None
        except Exception:
            sel = None
        self.sel = sel

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="qsa_clocks_", suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.sel:
            cmd += ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.remove(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup(ngpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=300))
    if ngpus != world:
        if rank == 0:
            print(f"warning: --gpus {ngpus} but WORLD_SIZE {world}", file=sys.stderr)
    return rank, world, local


def rank_seed(w: synth.Workload, rank: int) -> int:
    """Each rank runs an independent sequence (weak scaling)."""
    return w.seed + 7 * rank


def aggregate_tokens_per_s(world: int, w: synth.Workload, ms_per_step_max: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's step time."""
    return world * w.B * w.T / (ms_per_step_max / 1e3)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------- algorithmic work models --

def sparse_tokens_per_row(T: int, r: int, kb: int) -> np.ndarray:
    """|S(t)| for p = t: 4 per selected complete block + the own block's
    (t % r + 1) tokens; min(kb, c + 1) blocks."""
    t = np.arange(T, dtype=np.int64)
    c = t // r
    nblk = np.minimum(kb, c + 1)
    return r * (nblk - 1) + (t % r) + 1


def prefill_work(w: synth.Workload) -> dict:
    T, B = w.T, w.B
    S = sparse_tokens_per_row(T, w.r, w.kb).astype(np.float64)
    c = (np.arange(T) // w.r).astype(np.float64)
    return {
        "pool_bytes": B * (T * w.Di * 2 + (T // w.r) * w.Di * 2),
        "index_flops": B * float(c.sum()) * 2 * w.Hi * w.Di,
        "index_pairs": B * float(c.sum()),
        "index_bytes": B * (T * w.Hi * w.Di * 2 + T * w.Hi * 4 + (T // w.r) * w.Di * 2
                            + T * w.kb * 4),
        "attn_bytes": B * (float(S.sum()) * w.Hkv * w.D * 2 * 2 + T * w.Hq * w.D * 2 * 2
                           + T * w.kb * 4),
        "attn_flops": B * float(S.sum()) * 4 * w.Hq * w.D,
        "dense_flops": B * 4.0 * (T * (T + 1) / 2) * w.Hq * w.D,
    }


def decode_work(w: synth.Workload, seqlens) -> dict:
    L = np.asarray(seqlens, np.int64)
    c = (L - 1) // w.r
    nblk = np.minimum(w.kb, c + 1)
    S = w.r * (nblk - 1) + ((L - 1) % w.r) + 1
    return {
        "index_bytes": float((c * w.Di * 2).sum() + len(L) * (w.Hi * w.Di * 2 + w.kb * 4)),
        "attn_bytes": float((S * w.Hkv * w.D * 2 * 2).sum() + len(L) * w.Hq * w.D * 4),
        "dense_bytes": float((L * w.Hkv * w.D * 2 * 2).sum()),
    }


# ------------------------------------------------------------- GPU runners --

class Prefill:
    """Device buffers and one pass of the QSA prefill path for a workload."""

    def __init__(self, qsa, w, x, device):
        self.qsa, self.w, self.x = qsa, w, x
        B, T = w.B, w.T
        self.kp = torch.empty(B, T // w.r, w.Di, dtype=BF, device=device)
        self.sel = torch.empty(B, T, w.kb, dtype=torch.int32, device=device)
        self.o = torch.empty_like(x["q"])
        self.ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(
            B, T, T // w.r, w.Hi, w.Di, w.r, w.budget), device)
        self.stream = torch.cuda.current_stream(device)

    def step(self, ev=None):
        q, w, x = self.qsa, self.w, self.x
        nvtx = torch.cuda.nvtx
        if ev:
            ev[0].record(self.stream)
        nvtx.range_push("qsa_pool")
        q.qsa_pool(x["k_idx"], self.kp, w.r, stream=self.stream)
        nvtx.range_pop()
        if ev:
            ev[1].record(self.stream)
        nvtx.range_push("qsa_index_topk")
        q.qsa_index_topk(x["q_idx"], x["w"], self.kp, self.sel, self.ws, w.r, w.budget,
                         stream=self.stream)
        nvtx.range_pop()
        if ev:
            ev[2].record(self.stream)
        nvtx.range_push("qsa_sparse_attn_prefill")
        q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], self.sel, self.o, w.r, w.budget,
                                  w.scale, stream=self.stream)
        nvtx.range_pop()
        if ev:
            ev[3].record(self.stream)

    LAUNCHES = 3  # pool, index_topk, sparse_attn (the index counter reset is a memset)


def events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def flush_l2(buf):
    buf.add_(1)


def time_prefill(run: Prefill, steps: int, warmup: int, world: int, device, flush=None,
                 clocks: Clocks | None = None):
    nvtx = torch.cuda.nvtx
    nvtx.range_push("warmup")
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize(device)
    nvtx.range_pop()
    per = [events(4) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(device)
    if clocks:
        clocks.start()
    t0, t1 = events(2)
    nvtx.range_push("timed")
    t0.record(run.stream)
    for k in range(steps):
        if flush is not None:
            flush_l2(flush)  # outside the step's own events
        run.step(per[k])
    t1.record(run.stream)
    torch.cuda.synchronize(device)
    nvtx.range_pop()
    barrier(world)
    clk = clocks.stop() if clocks else None
    if flush is None:
        total = t0.elapsed_time(t1)  # back-to-back steps
    else:  # the steps' own event pairs, recorded after each flush
        total = sum(e[0].elapsed_time(e[3]) for e in per)
    kern = {"pool": 0.0, "index_topk": 0.0, "sparse_attn": 0.0}
    for e in per:
        kern["pool"] += e[0].elapsed_time(e[1])
        kern["index_topk"] += e[1].elapsed_time(e[2])
        kern["sparse_attn"] += e[2].elapsed_time(e[3])
    kern = {k: v / steps for k, v in kern.items()}
    return total, kern, clk


def e2e_prefill(qsa, w, x, device, steps):
    """Through the public API with host buffers: every step copies its inputs
    from pinned host memory to the device, runs the three calls and copies its
    output back, all inside the timing.  Steps are pipelined the way a server
    streams requests: the upload of step k + 1 (copy stream) and the download
    of step k - 1 (a second copy stream) overlap the kernels of step k (two
    device input and output buffers; events order each buffer's reuse)."""
    names = ["q", "k", "v", "q_idx", "k_idx", "w"]
    host = {n: torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=True) for n in names}
    for n in names:
        host[n].copy_(x[n])
    dev = [{n: torch.empty_like(x[n]) for n in names} for _ in range(2)]
    runs = [Prefill(qsa, w, dev[i], device) for i in range(2)]
    for r in runs[1:]:  # one set of intermediate buffers: the kernels run in stream order
        r.kp, r.sel, r.ws = runs[0].kp, runs[0].sel, runs[0].ws
    s_c = runs[0].stream
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    out_host = torch.empty(runs[0].o.shape, dtype=BF, pin_memory=True)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out_host.numel() * out_host.element_size()
    ev = lambda: torch.cuda.Event()
    copied = [ev(), ev()]      # inputs of buffer i are on the device
    computed = [ev(), ev()]    # step in buffer i done (inputs free, output ready)
    drained = [ev(), ev()]     # output of buffer i is back on the host
    for i in range(2):
        computed[i].record(s_c)
        drained[i].record(s_out)

    def upload(k):
        i = k % 2
        s_in.wait_event(computed[i])  # the step that used this buffer has read its inputs
        with torch.cuda.stream(s_in):
            for n in names:
                dev[i][n].copy_(host[n], non_blocking=True)
        copied[i].record(s_in)

    def compute(k):
        i = k % 2
        s_c.wait_event(copied[i])
        s_c.wait_event(drained[i])    # the output buffer has been read back
        runs[i].step()
        computed[i].record(s_c)

    def download(k):
        i = k % 2
        s_out.wait_event(computed[i])
        with torch.cuda.stream(s_out):
            out_host.copy_(runs[i].o, non_blocking=True)
        drained[i].record(s_out)

    def run(n_steps, t0=None, t1=None):
        if t0 is not None:
            t0.record(s_in)
        upload(0)
        for k in range(n_steps):
            if k + 1 < n_steps:
                upload(k + 1)
            compute(k)
            download(k)
        if t1 is not None:
            t1.record(s_out)

    run(2)  # warm-up
    torch.cuda.synchronize(device)
    a, b = events(2)
    run(steps, a, b)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    del host, dev, runs, out_host
    torch.cuda.empty_cache()
    return ms, h2d, d2h


def time_call(fn, stream, reps, warm=1, flush=None):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    evs = [events(2) for _ in range(reps)]
    for e in evs:
        if flush is not None:
            flush_l2(flush)
        e[0].record(stream)
        fn()
        e[1].record(stream)
    torch.cuda.synchronize()
    return sum(e[0].elapsed_time(e[1]) for e in evs) / reps


def dense_peak(peaks, ms):
    """bf16 peak for a dense call: the burst figure for a call timed alone, the
    sustained one once the call itself runs for seconds."""
    return peaks["bf16_tflops_sustained"] if ms >= 1000.0 else peaks["bf16_tflops"]


def torch_sdpa_ms(x, w, stream, reps, warm, flush):
    """torch's fused causal attention (flash / cuDNN) on the same tensors, with
    the KV heads repeated to the query heads; context for the speed-up."""
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        qt = x["q"].transpose(1, 2)
        kt = x["k"].repeat_interleave(w.G, dim=2).transpose(1, 2)
        vt = x["v"].repeat_interleave(w.G, dim=2).transpose(1, 2)
        with sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.CUDNN_ATTENTION]):
            ms = time_call(lambda: torch.nn.functional.scaled_dot_product_attention(
                qt, kt, vt, is_causal=True, scale=w.scale), stream, reps, warm, flush)
        del qt, kt, vt
        torch.cuda.empty_cache()
        return ms
    except Exception as exc:  # no fused backend for this shape: report why
        return f"unavailable: {type(exc).__name__}"


def roof(achieved, peak, unit, bound, traffic=None):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak if peak else None, "traffic": traffic}


def l2_read_gbs(qsa, device, mib=64, reps=40):
    """L2-to-SM read bandwidth from the library's probe kernel (16-byte L2 loads
    over a buffer that stays in L2), the denominator for gathers that L2 serves."""
    buf = torch.ones(mib << 18, dtype=torch.float32, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    s = torch.cuda.current_stream(device)
    for _ in range(2):
        qsa.qsa_probe_l2_read(buf, reps, sink, stream=s)
    torch.cuda.synchronize()
    best = None
    for _ in range(5):
        e0, e1 = events(2)
        e0.record(s)
        qsa.qsa_probe_l2_read(buf, reps, sink, stream=s)
        e1.record(s)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    return (mib << 20) * reps / (best / 1e3) / 1e9


def kernel_report(w, kern_ms, peaks):
    wk = prefill_work(w)
    hbm = peaks["hbm_gbs"]
    tf = peaks["bf16_tflops_sustained"]
    rep = {}
    for name, ms in kern_ms.items():
        s = ms / 1e3
        if name == "pool":
            rep[name] = {"ms": ms, "GB/s": wk["pool_bytes"] / s / 1e9,
                         "frac_hbm": wk["pool_bytes"] / s / 1e9 / hbm}
        elif name == "index_topk":
            rep[name] = {"ms": ms, "TFLOP/s": wk["index_flops"] / s / 1e12,
                         "frac_tensor": wk["index_flops"] / s / 1e12 / tf,
                         "pairs_per_s": wk["index_pairs"] / s}
        elif name == "sparse_attn":
            # the gathered K/V bytes are mostly served by L2 (selections overlap),
            # so they are reported as a gather rate, not against the HBM peak;
            # a DRAM fraction comes only from measured DRAM bytes
            dram = MEASURED_TRAFFIC.get((w.name, name))
            rep[name] = {"ms": ms, "gather_GB/s": wk["attn_bytes"] / s / 1e9,
                         "TFLOP/s": wk["attn_flops"] / s / 1e12,
                         "frac_tensor": wk["attn_flops"] / s / 1e12 / tf,
                         "dram_GB/s": dram / s / 1e9 if dram else None,
                         "frac_hbm_measured": dram / s / 1e9 / hbm if dram else None,
                         "frac_l2_measured": (wk["attn_bytes"] / s / 1e9 / peaks["l2_gbs"]
                                              if peaks.get("l2_gbs") else None)}
    return rep, wk


# DRAM bytes (read + write) per launch of a kernel, from a single-pass ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of that kernel in this
# benchmark's own command; keyed by (workload, kernel).  An entry is valid only
# for the kernel version it was taken on: remove it when the kernel changes.
MEASURED_TRAFFIC = {
    ("prefill-1m", "index_topk"): 5.841e9 + 14.170e9,
    ("prefill-1m", "sparse_attn"): 555.43e9 + 4.305e9,
}


def dominant_roofline(w, kern_ms, peaks, traffic=None):
    wk = prefill_work(w)
    name = max(kern_ms, key=kern_ms.get)
    if traffic is None:
        traffic = MEASURED_TRAFFIC.get((w.name, name))
    s = kern_ms[name] / 1e3
    if name == "index_topk":
        r = roof(wk["index_flops"] / s / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s",
                 "tensor", traffic)
    elif name == "sparse_attn":
        r = roof(wk["attn_flops"] / s / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s",
                 "tensor", traffic)
    else:
        r = roof(wk["pool_bytes"] / s / 1e9, peaks["hbm_gbs"], "GB/s", "hbm", traffic)
    r["kernel"] = name
    r["peak_source"] = peaks["source"]
    return r


# ------------------------------------------------------- secondary workloads

def extra_prefill(qsa, name, device, peaks, flush):
    w = synth.WORKLOADS[name]
    x = synth.make_prefill(w, device)
    run = Prefill(qsa, w, x, device)
    total, kern, _ = time_prefill(run, 5, 3, 1, device, flush=flush)
    ms = total / 5
    warm_total, _, _ = time_prefill(run, 5, 1, 1, device)  # no flush between steps
    warm_ms = warm_total / 5
    o = torch.empty_like(x["q"])
    dense = time_call(lambda: qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale),
                      run.stream, 2, 1, flush)
    rep, wk = kernel_report(w, kern, peaks)
    sdpa = torch_sdpa_ms(x, w, run.stream, 2, 1, flush)
    out = {"ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms / 1e3), "kernels": rep,
           "ms_per_step_warm": warm_ms,
           "torch_sdpa_dense_ms": sdpa,
           "dense_gqa_ms": dense,
           "dense_gqa_tflops": wk["dense_flops"] / (dense / 1e3) / 1e12,
           "dense_frac_tensor": wk["dense_flops"] / (dense / 1e3) / 1e12 / dense_peak(peaks, dense),
           "speedup_vs_torch_sdpa": sdpa / ms if isinstance(sdpa, float) else None,
           "speedup_vs_own_dense": dense / ms, "l2": "flushed between iterations"}
    del x, run, o
    torch.cuda.empty_cache()
    return out


def extra_decode(qsa, device, peaks, flush):
    w = synth.WORKLOADS["decode-256k-b64"]
    x = synth.make_decode(w, device)
    B, L = w.B, w.T
    kp = torch.empty(B, L // w.r, w.Di, dtype=BF, device=device)
    qsa.qsa_pool(x["k_idx_cache"], kp, w.r)
    sel = torch.empty(B, w.kb, dtype=torch.int32, device=device)
    o = torch.empty_like(x["q"])
    wsi = qsa.workspace(qsa.qsa_index_topk_decode_workspace_size(B, L // w.r, w.r, w.budget),
                        device)
    wsa = qsa.workspace(qsa.qsa_sparse_attn_decode_workspace_size(B, w.Hq, w.D, w.r, w.budget),
                        device)
    wsd = qsa.workspace(qsa.qsa_dense_gqa_decode_workspace_size(B, L, w.Hq, w.D), device)
    s = torch.cuda.current_stream(device)
    idx = lambda: qsa.qsa_index_topk_decode(x["q_idx"], x["w"], kp, x["seqlens"], sel, wsi,
                                            w.r, w.budget, stream=s)
    att = lambda: qsa.qsa_sparse_attn_decode(x["q"], x["k_cache"], x["v_cache"], x["seqlens"],
                                             sel, o, wsa, w.r, w.budget, w.scale, stream=s)

    def step():
        idx()
        att()

    t_step = time_call(step, s, 20, 3, flush)
    t_idx = time_call(idx, s, 20, 1, flush)
    t_att = time_call(att, s, 20, 1, flush)
    t_dense = time_call(lambda: qsa.qsa_dense_gqa_decode(x["q"], x["k_cache"], x["v_cache"],
                                                         x["seqlens"], o, wsd, w.scale, stream=s),
                        s, 5, 1, flush)
    wk = decode_work(w, x["seqlens"].cpu().numpy())
    hbm = peaks["hbm_gbs"]
    out = {
        "us_per_step": t_step * 1e3, "us_per_token": t_step * 1e3 / B, "batch": B,
        "cache_len": L,
        "kernels": {
            "index_topk_decode": {"us": t_idx * 1e3,
                                  "GB/s": wk["index_bytes"] / (t_idx / 1e3) / 1e9,
                                  "frac_hbm": wk["index_bytes"] / (t_idx / 1e3) / 1e9 / hbm},
            "sparse_attn_decode": {"us": t_att * 1e3,
                                   "GB/s": wk["attn_bytes"] / (t_att / 1e3) / 1e9,
                                   "frac_hbm": wk["attn_bytes"] / (t_att / 1e3) / 1e9 / hbm},
        },
        "step_frac_hbm": (wk["index_bytes"] + wk["attn_bytes"]) / (t_step / 1e3) / 1e9 / hbm,
        "dense_gqa_us": t_dense * 1e3,
        "dense_frac_hbm": wk["dense_bytes"] / (t_dense / 1e3) / 1e9 / hbm,
        "speedup_vs_dense": t_dense / t_step, "l2": "flushed between iterations",
        "launches_per_step": 4,
    }
    del x, kp
    torch.cuda.empty_cache()
    return out


def extra_gdn(qsa, device, flush):
    """The hybrid's other token mixer (gated delta rule) on one 16K-token sequence
    with 16 heads of 128 x 128 state: the exact recurrence and the chunked form,
    same inputs (unit keys, decay gates in [0.9, 1], write gates in [0, 1])."""
    B, T, H, dk, dv = 1, 16384, 16, 128, 128
    g = torch.Generator(device=device).manual_seed(7)
    q = torch.randn(B, T, H, dk, generator=g, device=device).to(BF)
    k = torch.randn(B, T, H, dk, generator=g, device=device)
    k = (k / k.norm(dim=-1, keepdim=True)).to(BF)
    v = torch.randn(B, T, H, dv, generator=g, device=device).to(BF)
    a = 0.9 + 0.1 * torch.rand(B, T, H, generator=g, device=device)
    b = torch.rand(B, T, H, generator=g, device=device)
    s0 = torch.randn(B, H, dv, dk, generator=g, device=device) * 0.1
    o1, o2 = (torch.empty(B, T, H, dv, device=device) for _ in range(2))
    s1, s2 = (torch.empty(B, H, dv, dk, device=device) for _ in range(2))
    ws = qsa.workspace(qsa.qsa_gdn_prefill_chunked_workspace_size(B, T, H, dk, dv), device)
    st = torch.cuda.current_stream(device)
    t_rec = time_call(lambda: qsa.qsa_gdn_prefill(q, k, v, a, b, o1, s1, state_in=s0, stream=st),
                      st, 3, 1, flush)
    t_chk = time_call(lambda: qsa.qsa_gdn_prefill_chunked(q, k, v, a, b, o2, s2, ws, state_in=s0,
                                                          stream=st), st, 5, 1, flush)
    diff = float((o1 - o2).abs().max() / o1.abs().max())
    out = {"shape": {"B": B, "T": T, "H": H, "dk": dk, "dv": dv}, "recurrence_ms": t_rec,
           "chunked_ms": t_chk, "speedup_chunked": t_rec / t_chk,
           "tokens_per_s_chunked": B * T / (t_chk / 1e3),
           "max_abs_diff_over_max": diff, "l2": "flushed between iterations"}
    del ws
    torch.cuda.empty_cache()
    return out


def extra_distill(qsa, device, peaks, flush):
    """Stage-1 indexer distillation (qsa_index_distill) at 32K tokens: the dense
    forward's lse and the pooled keys are made once, outside the timed call."""
    w = synth.WORKLOADS["prefill-32k"]
    x = synth.make_prefill(w, device)
    B, T, N = w.B, w.T, w.T // w.r
    f32 = dict(dtype=torch.float32, device=device)
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, T, w.Hq, **f32)
    qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale, lse=lse)
    kp = torch.empty(B, N, w.Di, dtype=BF, device=device)
    qsa.qsa_pool(x["k_idx"], kp, w.r)
    kl = torch.empty(B, T, **f32)
    dq = torch.empty(B, T, w.Hi, w.Di, **f32)
    dw = torch.empty(B, T, w.Hi, **f32)
    dkp = torch.empty(B, N, w.Di, **f32)
    dki = torch.empty(B, T, w.Di, **f32)
    ws = qsa.workspace(qsa.qsa_index_distill_workspace_size(B, T, w.Hkv, w.r), device)
    s = torch.cuda.current_stream(device)
    call = lambda: qsa.qsa_index_distill(x["q"], x["k"], lse, x["q_idx"], x["w"], kp, kl, dq,
                                         dw, dkp, ws, w.r, w.scale, dk_idx=dki, stream=s)
    ms = time_call(call, s, 3, 1, flush)
    status = qsa.qsa_check_device_status(ws)
    cpu = distill_oracle_sample(w, x, 16, seed=7)
    # teacher: 2 Hq D FLOP per (query, key) pair over the candidate blocks' keys;
    # indexer side: per (row, block) pair the scores (2 Hi Di), and the dq_idx and
    # dKp products (2 Hi Di each)
    teacher_flops = 2.0 * w.Hq * w.D * sum_candidate_keys(T, w.r)
    pairs = sum_candidate_keys(T, w.r) / w.r
    flops = teacher_flops + pairs * 3 * 2 * w.Hi * w.Di
    achieved = flops / (ms / 1e3) / 1e12
    out = {"workload": w.name, "ms": ms, "status": status,
           "teacher_flops": teacher_flops,
           "teacher_tflops_if_whole_call": teacher_flops / (ms / 1e3) / 1e12,
           "roofline": dict(roof(achieved, peaks["bf16_tflops"], "TFLOP/s", "tensor"),
                            scope="whole call, algorithmic FLOPs (teacher + indexer side)"),
           "row_block_pairs": pairs, "kl_mean": float(kl.mean()),
           "cpu_baseline": cpu,
           "finite": bool(torch.isfinite(dq).all() and torch.isfinite(dkp).all()),
           "l2": "flushed between iterations"}
    del x, o, lse, kp, kl, dq, dw, dkp, dki, ws
    torch.cuda.empty_cache()
    return out


def distill_oracle_sample(w: synth.Workload, x: dict, n_rows: int, seed: int) -> dict:
    """The distillation oracle (numpy, fp64) on stratified rows of the workload;
    the mean time per row, times T, estimates one whole call."""
    from oracle import distill  # test/baseline infrastructure only
    import oracle
    host = {n: oracle.bf16_bits_to_f64(synth.bf16_bits(x[n])[0])
            for n in ("q", "k", "q_idx", "k_idx")}
    kp = oracle.bf16_bits_to_f64(oracle.pool(synth.bf16_bits(x["k_idx"]), w.r)[0])
    wt = x["w"][0].cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, w.T, n_rows + 1).astype(np.int64)
    rows = np.array([rng.integers(edges[i], max(edges[i] + 1, edges[i + 1]))
                     for i in range(n_rows)], np.int64)
    t0 = time.perf_counter()
    distill.distill_rows_f64(host["q"], host["k"], host["q_idx"], wt, kp, w.r, w.scale,
                             rows=rows)
    secs = time.perf_counter() - t0
    est_ms = secs / n_rows * w.T * 1e3
    return {"value": est_ms, "unit": "ms per call (extrapolated)", "cores": cpu_cores(),
            "kind": "oracle",
            "sample": f"{n_rows} stratified query rows of {w.name}, {secs:.1f} s wall; mean "
                      f"time per row times {w.T} rows"}


def sum_candidate_keys(T: int, r: int) -> float:
    """Sum over query rows p < T of r * floor(p / r): the keys of every row's
    candidate blocks (exact integer arithmetic)."""
    m, rem = divmod(T, r)           # rows p = r*c + i: m full groups, then rem rows of c = m
    full = r * r * (m * (m - 1) // 2)  # sum over c < m of r rows x r*c keys
    return float(full + rem * r * m)


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(w: synth.Workload, x: dict, n_rows: int, seed: int, threads: int | None = None):
    """Time the CPU oracle on stratified query rows of the workload.

    Rows are drawn one per equal-width stratum of [0, T) so that their mean
    cost estimates the mean over all rows; pooling is timed over the whole
    sequence and charged per token.  Returns (tokens/s, seconds, rows)."""
    import oracle  # test/baseline infrastructure only
    if threads:
        oracle.set_num_threads(threads)
    host = {n: synth.bf16_bits(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    wt = x["w"].cpu().numpy()
    t0 = time.perf_counter()
    kp = oracle.pool(host["k_idx"], w.r)
    t_pool = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, w.T, n_rows + 1).astype(np.int64)
    rows = np.array([rng.integers(edges[i], max(edges[i] + 1, edges[i + 1]))
                     for i in range(n_rows)], np.int64)
    t0 = time.perf_counter()
    sel, _, _, _ = oracle.index_topk(host["q_idx"], wt, kp, w.r, w.budget, rows=rows)
    oracle.attn(host["q"], host["k"], host["v"], w.r, w.scale, sel=sel, rows=rows)
    t_rows = time.perf_counter() - t0
    per_token = t_rows / n_rows + t_pool / (w.B * w.T)
    return 1.0 / per_token, t_rows + t_pool, rows.size


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# -------------------------------------------------------------------- main --

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    device = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.make_prefill(w, device)
    import oracle
    cores = oracle.num_threads()
    n_rows = args.ref_rows
    for k in range(args.warmup):
        oracle_sample(w, x, max(8, n_rows // 4), seed=1000 + k)
    vals, secs = [], []
    for k in range(args.steps):
        v, s, _ = oracle_sample(w, x, n_rows, seed=k)
        vals.append(v)
        secs.append(s)
    value = len(vals) / sum(1.0 / v for v in vals)  # tokens over total time
    sample = (f"{n_rows} stratified query rows of the {w.name} workload per step "
              f"(index top-k + attention per row, pooling charged per token), "
              f"rows/s extrapolated to tokens/s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(secs) / len(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, l2_label(w, x)),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def input_bytes(x) -> int:
    return sum(x[n].numel() * x[n].element_size() for n in ("q", "k", "v", "q_idx", "k_idx", "w"))


def l2_label(w, x) -> str:
    b = input_bytes(x)
    return ("L2 flushed between steps" if b < 4 * L2_BYTES else
            f"inputs larger than L2 ({b / 1e9:.1f} GB per step)")


def config_of(w, l2):
    return {"workload": w.name, "batch": w.B, "seq_len": w.T, "q_heads": w.Hq,
            "kv_heads": w.Hkv, "head_dim": w.D, "indexer_heads": w.Hi, "indexer_dim": w.Di,
            "block": w.r, "token_budget": w.budget, "seed": w.seed, "l2": l2}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="qsa", choices=["qsa", "reference"])
    ap.add_argument("--workload", default="prefill-1m",
                    choices=[n for n, w in synth.WORKLOADS.items() if w.kind == "prefill"])
    ap.add_argument("--no-extra", action="store_true", help="skip the 128K, decode and distillation lines")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense GQA ratio run")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--cpu-rows", type=int, default=256)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    import block_sparse_long_10_b200 as qsa
    qsa.load()  # fails loudly if the CUDA library is missing
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks = load_peaks()
    peaks["l2_gbs"] = l2_read_gbs(qsa, device)
    w = synth.WORKLOADS[args.workload]
    seed = rank_seed(w, rank)
    x = synth.make_prefill(w, device, seed=seed)
    in_bytes = input_bytes(x)
    run = Prefill(qsa, w, x, device)
    flush = None
    if in_bytes < 4 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    clocks = Clocks(local)
    total_ms, kern, clk = time_prefill(run, args.steps, args.warmup, world, device,
                                       flush=flush, clocks=clocks)
    total_ms = max_over_ranks(total_ms, world, device)
    ms_step = total_ms / args.steps
    value = aggregate_tokens_per_s(world, w, ms_step)
    kern_rep, wk = kernel_report(w, kern, peaks)
    roofline = dominant_roofline(w, kern, peaks)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, l2_label(w, x)),
        "roofline": roofline, "kernels": kern_rep,
        "l2_probe": {"GB/s": peaks["l2_gbs"], "bytes": 64 << 20, "reps": 40,
                     "note": "qsa_probe_l2_read: 16-byte L2 loads on all SMs over a 64 MiB "
                             "buffer; the sparse attention's gather rate is also given as a "
                             "fraction of it"},
        "gpu_launches": Prefill.LAUNCHES * args.steps,
        "clocks": clk,
    }
    barrier(world)
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_prefill(qsa, w, x, device, args.steps)
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        line["e2e"] = {"value": world * w.B * w.T / (e2e_ms / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_ms,
                       "note": "public API, pinned host buffers; each step's upload and "
                               "download overlap the neighbouring steps' kernels "
                               "(two copy streams, two device buffer sets)"}
    barrier(world)
    if rank == 0:
        if not args.no_dense:
            o = torch.empty_like(x["q"])
            if w.T >= 2**19:  # load the kernel on a short prefix first
                qsa.qsa_dense_gqa_prefill(x["q"][:, :4096].contiguous(),
                                          x["k"][:, :4096].contiguous(),
                                          x["v"][:, :4096].contiguous(),
                                          o[:, :4096].contiguous(), w.scale)
            d_ms = time_call(lambda: qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale),
                             run.stream, 1, 0 if w.T >= 2**19 else 1, flush)
            del o
            torch.cuda.empty_cache()
            sdpa = torch_sdpa_ms(x, w, run.stream, 1, 1, flush)
            line["dense_gqa"] = {
                "torch_sdpa_ms": sdpa,
                "speedup_qsa_vs_torch_sdpa": sdpa / ms_step if isinstance(sdpa, float) else None,
                "own_kernel_ms": d_ms,
                "own_kernel_tflops": wk["dense_flops"] / (d_ms / 1e3) / 1e12,
                "own_kernel_frac_tensor": wk["dense_flops"] / (d_ms / 1e3) / 1e12
                / dense_peak(peaks, d_ms),
                "speedup_qsa_vs_own_kernel": d_ms / ms_step,
                "note": "torch SDPA (flash / cuDNN) is the main dense comparison; the "
                        "library's own dense kernel is secondary"}
        if not args.no_cpu and world == 1:
            import oracle  # test/baseline infrastructure only
            threads = oracle.num_threads()
            v, secs, n = oracle_sample(w, x, args.cpu_rows, seed=12345)
            v1, secs1, n1 = oracle_sample(w, x, max(8, args.cpu_rows // 8), seed=54321,
                                          threads=1)
            oracle.set_num_threads(threads)
            line["cpu_baseline"] = {
                "value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": f"{n} stratified query rows of {w.name} (index top-k + attention "
                          f"per row) plus pooling of the whole sequence, {secs:.1f} s wall; "
                          f"rows/s extrapolated to tokens/s",
                "one_thread": {"value": v1, "unit": "tokens/s", "cores": 1,
                               "sample": f"{n1} stratified rows, {secs1:.1f} s wall"}}
        if not args.no_extra:
            del run
            torch.cuda.empty_cache()
            fl = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
            line["extra"] = {}
            if w.name != "prefill-128k":
                line["extra"]["prefill-128k"] = extra_prefill(qsa, "prefill-128k", device, peaks, fl)
            line["extra"]["decode-256k-b64"] = extra_decode(qsa, device, peaks, fl)
            try:  # a secondary measurement: report a failure instead of losing the line
                line["extra"]["distill-32k"] = extra_distill(qsa, device, peaks, fl)
            except Exception as exc:
                line["extra"]["distill-32k"] = {"error": f"{type(exc).__name__}: {exc}"}
            try:
                line["extra"]["gdn-16k-h16"] = extra_gdn(qsa, device, fl)
            except Exception as exc:
                line["extra"]["gdn-16k-h16"] = {"error": f"{type(exc).__name__}: {exc}"}
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
