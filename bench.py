"""Benchmark of the GDN hot path on B200: prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (`value`): GDN chunkwise prefill tokens/s on the long-context
Qwen3.5-shaped layer (B=1, T=131072, 16 key heads, 64 value heads, d=128, bf16
inputs, fp32 state), the largest configuration that runs on one GPU; one step =
one gdn_chunk_fwd call over that batch: two kernels, a chunk-parallel WY prep
(gates, L2 norm, K K^T / Q K^T, (I+L)^-1, W, U, A_qk) and the scan over chunks
(U - W S, output rows, state update).  `e2e` is the same workload through the
host entry point (gdn_chunk_fwd_host) with page-locked host inputs and outputs,
every copy inside the timed region.  The 8K-token prefill, the batched 8 x 16K
prefill, the decode step (256 sequences, fused conv1d, state GB/s), the Gated
DeltaNet-2 and KDA forwards, the prefill conv and the gated RMSNorm are measured
in the same run and reported under "extra".  Multi-GPU runs are independent
replicas (every (batch, head) scan is independent; no collective on the data
path): weak scaling, time = max over ranks.  `--impl reference` times the fp64
CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from gdn_synth import WORKLOADS, kda_inputs, workload_inputs  # noqa: E402

# dense GEMM FLOPs of the chunk form at C=64, d=128 per token and value head
# (10 C d + 6 d^2); with the K K^T / Q K^T Gram formed once per key head and shared
# by a GQA group of G = 4 value heads, the work the kernels need is 155,648
CHUNK_FLOP_PER_TOKEN_HEAD = 180_224
CHUNK_FLOP_PER_TOKEN_HEAD_GQA4 = 155_648
HEADLINE = "prefill_128k"


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "src": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        rows = [l for (t, l) in self.lines if t0 - 0.06 <= t <= t1 + 0.06] or \
            [l for (_, l) in self.lines[-3:]]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            f = [x.strip() for x in l.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def flush_l2(buf):
    buf.add_(1.0)


def rank_info():
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) > 1:
        return int(os.environ["RANK"]), int(os.environ["LOCAL_RANK"]), int(os.environ["WORLD_SIZE"])
    return 0, 0, 1


def max_over_ranks(x: float, device) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes units_per_rank per step (weak
    scaling, independent replicas), the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_per_step / 1e3)


def kernel_traffic(name):
    """dram bytes per launch from a committed ncu summary, if the kernel sources it
    lists (`source_files:`, relative to the package's csrc/; every source when the
    line is absent) still hash to its `source_sha256` (else None)."""
    path = os.path.join(ROOT, "profiles", f"{name}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{16,64})", txt)
    f = re.search(r"source_files:\s*(.+)", txt)
    if not m or not h:
        return None
    files = f.group(1).split() if f else None
    return float(m.group(1)) if h.group(1) == source_hash(files)[:len(h.group(1))] else None


def source_hash(files=None):
    """sha256 over the given kernel sources (names in csrc/, in the given order), or
    over every .cu / .cuh / .h of csrc/ in name order."""
    d = os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "csrc")
    if files is None:
        files = sorted(f for f in os.listdir(d) if f.endswith((".cu", ".cuh", ".h")))
    hs = hashlib.sha256()
    for f in files:
        hs.update(open(os.path.join(d, f), "rb").read())
    return hs.hexdigest()


# ----------------------------------------------------------------------------- our arm
def time_steps(fn, steps, warmup, stream, flush=None, sync_group=False):
    """CUDA-event time of `steps` calls of fn on `stream`, after `warmup` calls.
    Returns (total_ms, per-launch ms list)."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    if sync_group:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(steps):
            if flush is not None:
                flush()
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize()
    if sync_group:
        dist.barrier()
    per = [a.elapsed_time(b) for a, b in evs]
    return start.elapsed_time(end), per


def prefill_roofline(w, launch_ms, pk, profile):
    """Roofline of one gdn_chunk_fwd call on workload w: the dense GEMM FLOPs of
    the chunk form (and, beside them, the GQA-shared count) over the call's mean
    CUDA-event time, against the measured bf16 burst peak."""
    flop = CHUNK_FLOP_PER_TOKEN_HEAD * w.T * w.Hv * w.B
    flop_gqa = CHUNK_FLOP_PER_TOKEN_HEAD_GQA4 * w.T * w.Hv * w.B
    achieved = flop / (launch_ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2),
            "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / pk["bf16_tflops"], 4),
            "traffic": kernel_traffic(profile),
            "kernel": "gdn_chunk_fwd = wy_prep_tc_kernel + state_scan_tc_kernel (timed together)",
            "flop_per_launch": flop,
            "frac_gqa_shared_count": round(flop_gqa / (launch_ms / 1e3) / 1e12
                                           / pk["bf16_tflops"], 4),
            "flop_per_launch_gqa_shared": flop_gqa,
            "peak_src": pk["src"] + " burst bf16"}


def run_ours(args, rank, local_rank, world):
    import gated_deltanet_sequence_gdn_b200 as G

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    pk = peaks()
    w = WORKLOADS[HEADLINE]
    x = workload_inputs(w, dev)
    o = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)
    ht = torch.empty((w.B, w.Hv, w.d, w.d), device=dev, dtype=torch.float32)
    ws = chunk_workspace(G, w, dev)

    def step():
        G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"], o=o, ht=ht, workspace=ws, stream=stream)

    clocks = ClockSampler(local_rank).start()
    time.sleep(0.3)
    t0 = time.time()
    total_ms, per = time_steps(step, args.steps, args.warmup, stream, sync_group=world > 1)
    t1 = time.time()
    clk = clocks.stop(t0, t1)
    G.gdn_check_status(stream)
    ms_step = max_over_ranks(total_ms, dev) / args.steps
    tokens = w.B * w.T
    value = job_rate(tokens, world, ms_step)
    launch_ms = sum(per) / len(per)
    roofline = prefill_roofline(w, launch_ms, pk, "chunk_prefill_128k")
    del ws, o, ht
    torch.cuda.empty_cache()

    # ---- end to end through the public call, host buffers, copies inside the timed region
    e2e = measure_e2e(G, x, w, dev, stream, args, world)
    x_cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x_cpu = {n: (t.cpu() if t is not None else None) for n, t in x.items()}
    del x
    torch.cuda.empty_cache()

    extra = {}
    if not args.headline_only:
        extra["prefill_8k"] = measure_prefill(G, "prefill_8k", dev, stream, pk, args)
        extra["prefill_b8_16k"] = measure_prefill(G, "prefill_b8_16k", dev, stream, pk, args)
        extra["decode_256"] = measure_decode(G, dev, stream, pk, args)
        extra["gdn2_b4_4k"] = measure_gdn2(G, dev, stream, pk, args)
        extra["conv_prefill_8k"] = measure_conv(G, dev, stream, pk, args)
        extra["gate_prep_8k"] = measure_gate_prep(G, dev, stream, pk, args)
        extra["prefill_8k_gated_norm"] = measure_prefill_gated_norm(G, dev, stream, pk, args)
        # the newest secondary figures, last: a failure is reported here, not raised
        for name, fn in (("kda_b4_4k", measure_kda), ("rmsnorm_gated_8k", measure_norm),
                         ("bwd_8k", measure_bwd)):
            try:
                extra[name] = fn(G, dev, stream, pk, args)
                torch.cuda.synchronize()
            except Exception as e:  # noqa: BLE001
                extra[name] = {"error": f"{type(e).__name__}: {e}"[:300]}

    launches = 2 * args.steps  # wy_prep_tc_kernel + state_scan_tc_kernel per step
    line = {
        "metric": "GDN prefill tokens/s (chunk_gated_delta_rule) on 1 B200, % of roofline",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": HEADLINE, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv,
                   "d": w.d, "chunk": 64, "state": "fp32", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (q,k,v,o ~5.4 GB per step > 126 MB)"},
        "roofline": roofline, "e2e": e2e, "clocks": clk, "gpu_launches": launches,
        "extra": extra,
    }
    if x_cpu is not None:
        line["cpu_baseline"] = cpu_baseline(w, x_cpu)
    return line


def chunk_workspace(G, w, dev):
    n = G.gdn_chunk_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.d, w.d, w.dtype)
    return torch.empty(n, device=dev, dtype=torch.uint8) if n > 0 else None


def measure_e2e(G, x, w, dev, stream, args, world):
    """The headline metric end to end: page-locked host inputs in, host outputs
    out, through the library's host entry point (gdn_chunk_fwd_host), which
    pipelines the host link and the kernels piece by piece; every copy is
    inside the timed region."""
    host = {n: (t.cpu().pin_memory() if t is not None else None) for n, t in x.items()}
    o_h = torch.empty((w.B, w.T, w.Hv, w.d), dtype=w.dtype).pin_memory()
    ht_h = torch.empty((w.B, w.Hv, w.d, w.d), dtype=torch.float32).pin_memory()
    need = G.gdn_chunk_fwd_host_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.d, w.d, w.dtype)
    dws = torch.empty(need, device=dev, dtype=torch.uint8)
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = o_h.numel() * o_h.element_size() + ht_h.numel() * ht_h.element_size()

    def step():
        G.gdn_chunk_fwd_host(host["q"], host["k"], host["v"], host["a"], host["b"],
                             host["A_log"], host["dt_bias"], host["h0"], o=o_h, ht=ht_h,
                             dev_workspace=dws, stream=stream, sync=False)

    piece = max(64, (((w.T + 7) // 8 + 63) // 64) * 64)
    steps = max(3, min(args.steps, 20))
    total_ms, _ = time_steps(step, steps, 2, stream, sync_group=world > 1)
    ms_step = max_over_ranks(total_ms, dev) / steps
    return {"value": round(job_rate(w.B * w.T, world, ms_step), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms_step, 4), "steps": steps,
            "path": "pinned host -> gdn_chunk_fwd_host (C ABI; copies in, kernels and copies "
                    f"out pipelined over pieces of {piece} tokens, the default T/8 in whole "
                    "chunks) -> pinned host"}


def measure_prefill(G, name, dev, stream, pk, args):
    w = WORKLOADS[name]
    x = workload_inputs(w, dev)
    o = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)
    ht = torch.empty((w.B, w.Hv, w.d, w.d), device=dev, dtype=torch.float32)
    ws = chunk_workspace(G, w, dev)

    def step():
        G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"], o=o, ht=ht, workspace=ws, stream=stream)

    steps = 10 if w.T * w.B <= 16384 else 5
    total, per = time_steps(step, steps, 3, stream)
    ms = sum(per) / len(per)
    rl = prefill_roofline(w, ms, pk, "chunk_" + name)
    del x, o, ht, ws
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "B": w.B, "T": w.T, "achieved_tflops": rl["achieved"],
            "frac_of_bf16_peak": rl["frac"], "roofline": rl, "steps": steps}


def measure_decode(G, dev, stream, pk, args):
    w = WORKLOADS["decode_256"]
    x = workload_inputs(w, dev)
    cs, S = x["conv_state"], x["state"]
    o = torch.empty((w.B, w.Hv, w.d), device=dev, dtype=w.dtype)
    it = [0]

    def step():
        t = it[0] % w.steps
        it[0] += 1
        G.gdn_recurrent_step(x["x"][t], x["conv_w"], cs, x["a"][t], x["b"][t], x["A_log"],
                             x["dt_bias"], S, Hk=w.Hk, Hv=w.Hv, dk=w.d, dv=w.d, o=o,
                             stream=stream)

    total, per = time_steps(step, w.steps, 3, stream)
    ms = total / w.steps
    state_bytes = 2 * w.B * w.Hv * w.d * w.d * 4
    Cc = 2 * w.Hk * w.d + w.Hv * w.d
    other = w.B * Cc * 2 + 2 * w.B * Cc * 3 * 2 + Cc * 16 + w.B * w.Hv * (4 + w.d * 2)
    gbs = state_bytes / (ms / 1e3) / 1e9
    del x, cs, S
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B / (ms / 1e3), 1), "ms_per_step": round(ms, 5),
            "state_gb_per_s": round(gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": state_bytes,
                         "other_bytes_per_launch": other,
                         "traffic": kernel_traffic("decode_256")},
            "steps": w.steps}


def measure_gdn2(G, dev, stream, pk, args):
    w = WORKLOADS["gdn2_b4_4k"]
    x = workload_inputs(w, dev)
    o = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)
    ht = torch.empty((w.B, w.Hv, w.d, w.d), device=dev, dtype=torch.float32)
    n_ws = G.gdn2_chunk_workspace_bytes(w.B, w.T, w.Hv, w.d, w.d, w.dtype)
    ws = torch.empty(n_ws, device=dev, dtype=torch.uint8) if n_ws else None

    def step():
        G.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b_logit"], x["w_logit"],
                         x["A_log"], x["dt_bias"], x["h0"], o=o, ht=ht, workspace=ws,
                         stream=stream)

    total, per = time_steps(step, 5, 2, stream)
    ms = total / 5
    flop = CHUNK_FLOP_PER_TOKEN_HEAD * w.T * w.Hv * w.B
    ach = flop / (ms / 1e3) / 1e12
    del x, o, ht, ws
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "achieved_tflops": round(ach, 2),
            "frac_of_bf16_peak": round(ach / pk["bf16_tflops"], 4)}


def measure_conv(G, dev, stream, pk, args):
    """gdn_conv_prefill over the mixed stream of the prefill_8k layer: HBM-bound,
    reported against the measured copy bandwidth.  Algorithmic bytes per launch:
    the input stream read once, q, k, v written once, the taps and the window read
    and written (inputs of 201 MB, larger than L2, so no flush between launches)."""
    w = WORKLOADS["conv_prefill_8k"]
    x = workload_inputs(w, dev)
    Cc = 2 * w.Hk * w.d + w.Hv * w.d
    cs = x["conv_state"]
    q = torch.empty((w.B, w.T, w.Hk, w.d), device=dev, dtype=w.dtype)
    k = torch.empty_like(q)
    v = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)

    def step():
        G.gdn_conv_prefill(x["x"], x["conv_w"], cs, Hk=w.Hk, Hv=w.Hv, dk=w.d, dv=w.d, q=q, k=k,
                           v=v, stream=stream)

    steps = 20
    total, per = time_steps(step, steps, 3, stream)
    ms = sum(per) / len(per)
    es = 2  # bf16
    nbytes = 2 * w.B * w.T * Cc * es + Cc * 16 + 2 * w.B * Cc * 3 * es
    gbs = nbytes / (ms / 1e3) / 1e9
    del x, cs, q, k, v
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_launch": round(ms, 5),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": kernel_traffic("conv_prefill_8k")},
            "steps": steps}


def measure_gate_prep(G, dev, stream, pk, args):
    """gdn_gate_prep over the prefill_8k layer (q, k [1, 8192, 16, 128] bf16 and the
    gate inputs of 64 value heads): HBM-bound.  Algorithmic bytes per launch: q, k
    read and q_hat, k_hat written once (bf16), a, b read (bf16), g, beta written
    (float32), A_log / dt_bias read."""
    w = WORKLOADS["prefill_8k"]
    x = workload_inputs(w, dev)
    qo, ko = torch.empty_like(x["q"]), torch.empty_like(x["k"])
    g = torch.empty((w.B, w.T, w.Hv), device=dev, dtype=torch.float32)
    beta = torch.empty_like(g)

    def step():
        G.gdn_gate_prep(x["q"], x["k"], x["a"], x["b"], x["A_log"], x["dt_bias"], q_out=qo,
                        k_out=ko, g_out=g, beta_out=beta, stream=stream)

    steps = 20
    total, per = time_steps(step, steps, 3, stream)
    ms = sum(per) / len(per)
    es = 2
    nbytes = (2 * 2 * w.B * w.T * w.Hk * w.d * es + 2 * w.B * w.T * w.Hv * es
              + 2 * w.B * w.T * w.Hv * 4 + 2 * w.Hv * 4)
    gbs = nbytes / (ms / 1e3) / 1e9
    del x, qo, ko, g, beta
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_launch": round(ms, 5),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": kernel_traffic("gate_prep_8k")},
            "steps": steps}


# Dense products of one gdn_chunk_bwd call per 64-token chunk and value head at
# d = 128, in multiply-adds: the chunk prep (K K^T, Q K^T, W, U: 4 C^2 d), the
# forward state scan (W S0, K~^T U~: 2 C d^2), the reverse scan (K~ dS, (gamma Q)^T
# dO, W^T dU~: 3 C d^2, A_qk^T dO: C^2 d) and the per-chunk gradients (dQ, dW, dK~,
# Q S0: 4 C d^2; dA_qk, dA twice, dVb, dKb, dKK K twice, dQK K, dQK^T Q: 9 C^2 d;
# dA A^T, A^T (.): 2 C^3) -> 2 (9 C d^2 + 14 C^2 d + 2 C^3) / C FLOP per token.
BWD_FLOP_PER_TOKEN_HEAD = 2 * (9 * 64 * 128 * 128 + 14 * 64 * 64 * 128 + 2 * 64 ** 3) // 64


def measure_bwd(G, dev, stream, pk, args):
    """gdn_chunk_bwd on the prefill_8k layer (the backward of one gdn_chunk_fwd call,
    output gradients ~ N(0,1)); float32 arithmetic on the CUDA cores, so its
    roofline is the fp32 FMA rate: 148 SMs x 128 lanes x 2 FLOP x the SM clock."""
    from gdn_synth import bwd_cotangents
    w = WORKLOADS["prefill_8k"]
    x = workload_inputs(w, dev)
    ct = bwd_cotangents(w.B, w.T, w.Hv, w.d, w.d, w.dtype, 1501, dev)
    ws = torch.empty(G.gdn_chunk_bwd_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.d, w.d),
                     device=dev, dtype=torch.uint8)

    def step():
        G.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"], ct["do"], ct["dht"], workspace=ws, stream=stream)

    steps = 3
    total, per = time_steps(step, steps, 3, stream)
    ms = sum(per) / len(per)
    flop = BWD_FLOP_PER_TOKEN_HEAD * w.B * w.T * w.Hv
    tf = flop / (ms / 1e3) / 1e12
    peak = 148 * 128 * 2 * 1965e6 / 1e12  # clocks.max.sm of this part: 1965 MHz
    del x, ct, ws
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_call": round(ms, 4),
            "roofline": {"bound": "alu", "achieved": round(tf, 2), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                         "flop_per_call": flop,
                         "peak_src": "fp32 FMA: 148 SMs x 128 lanes x 2 x max SM clock"},
            "steps": steps}


def measure_prefill_gated_norm(G, dev, stream, pk, args):
    """prefill_8k through gdn_chunk_fwd_gated_norm (the gated RMSNorm of the output
    stage fused into the scan's output store), beside gdn_chunk_fwd followed by the
    standalone gdn_rmsnorm_gated: the same result, one HBM pass over o and the
    norm's own kernel fewer."""
    w = WORKLOADS["prefill_8k"]
    x = workload_inputs(w, dev)
    g = torch.Generator(device="cpu").manual_seed(1008)
    z = torch.randn((w.B, w.T, w.Hv, w.d), generator=g).to(w.dtype).to(dev)
    nw = (0.5 + torch.rand(w.d, generator=g)).to(dev)
    o = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)
    y = torch.empty_like(o)
    ht = torch.empty((w.B, w.Hv, w.d, w.d), device=dev, dtype=torch.float32)
    ws = chunk_workspace(G, w, dev)

    def fused():
        G.gdn_chunk_fwd_gated_norm(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                   x["dt_bias"], x["h0"], z, nw, o=o, ht=ht, workspace=ws,
                                   stream=stream)

    def composed():
        G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"], o=o, ht=ht, workspace=ws, stream=stream)
        G.gdn_rmsnorm_gated(o, z, nw, y=y, stream=stream)

    _, per_f = time_steps(fused, 10, 3, stream)
    _, per_c = time_steps(composed, 10, 3, stream)
    ms_f, ms_c = sum(per_f) / len(per_f), sum(per_c) / len(per_c)
    rl = prefill_roofline(w, ms_f, pk, "chunk_prefill_8k_gated_norm")
    del x, z, o, y, ht, ws
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms_f / 1e3), 1), "ms_per_step": round(ms_f, 4),
            "ms_per_step_unfused": round(ms_c, 4), "frac_of_bf16_peak": rl["frac"],
            "roofline": rl}


def measure_kda(G, dev, stream, pk, args):
    """gdn_kda_chunk_fwd at the Gated DeltaNet-2 bench shape (B=4, T=4096, 16 heads,
    d=128, bf16): the gate tiling plus the Gated DeltaNet-2 kernels."""
    w = WORKLOADS["gdn2_b4_4k"]
    x = kda_inputs(w.B, w.T, w.Hv, w.d, w.dtype, seed=1007, device=dev)
    o = torch.empty((w.B, w.T, w.Hv, w.d), device=dev, dtype=w.dtype)
    ht = torch.empty((w.B, w.Hv, w.d, w.d), device=dev, dtype=torch.float32)
    n_ws = G.gdn_kda_chunk_workspace_bytes(w.B, w.T, w.Hv, w.d, w.d, w.dtype)
    ws = torch.empty(n_ws, device=dev, dtype=torch.uint8)

    def step():
        G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                            x["dt_bias"], x["h0"], o=o, ht=ht, workspace=ws, stream=stream)

    total, per = time_steps(step, 5, 2, stream)
    ms = total / 5
    flop = CHUNK_FLOP_PER_TOKEN_HEAD * w.T * w.Hv * w.B
    ach = flop / (ms / 1e3) / 1e12
    del x, o, ht, ws
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "achieved_tflops": round(ach, 2),
            "frac_of_bf16_peak": round(ach / pk["bf16_tflops"], 4)}


def measure_norm(G, dev, stream, pk, args):
    """gdn_rmsnorm_gated over the prefill_8k layer's core output (8192 tokens x 64
    value heads x 128): HBM-bound, reported against the measured copy bandwidth.
    Algorithmic bytes per launch: o and z read once, y written once, the weight."""
    w = WORKLOADS["rmsnorm_gated_8k"]
    x = workload_inputs(w, dev)
    y = torch.empty_like(x["o"])

    def step():
        G.gdn_rmsnorm_gated(x["o"], x["z"], x["weight"], y=y, stream=stream)

    steps = 20
    total, per = time_steps(step, steps, 3, stream)
    ms = sum(per) / len(per)
    nbytes = 3 * x["o"].numel() * x["o"].element_size() + w.d * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    del x, y
    torch.cuda.empty_cache()
    return {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_launch": round(ms, 5),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": kernel_traffic("rmsnorm_gated_8k")},
            "steps": steps}


def run_only(args, local_rank):
    import gated_deltanet_sequence_gdn_b200 as G
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    pk = peaks()
    if args.only == "decode_256":
        r = measure_decode(G, dev, stream, pk, args)
    elif args.only == "gdn2_b4_4k":
        r = measure_gdn2(G, dev, stream, pk, args)
    elif args.only == "conv_prefill_8k":
        r = measure_conv(G, dev, stream, pk, args)
    elif args.only == "rmsnorm_gated_8k":
        r = measure_norm(G, dev, stream, pk, args)
    elif args.only == "kda_b4_4k":
        r = measure_kda(G, dev, stream, pk, args)
    elif args.only == "gate_prep_8k":
        r = measure_gate_prep(G, dev, stream, pk, args)
    elif args.only == "prefill_8k_gated_norm":
        r = measure_prefill_gated_norm(G, dev, stream, pk, args)
    elif args.only == "bwd_8k":
        r = measure_bwd(G, dev, stream, pk, args)
    else:
        r = measure_prefill(G, args.only, dev, stream, pk, args)
    G.gdn_check_status(stream)
    return {"workload": args.only, **r}


# ----------------------------------------------------------------------------- oracle
def _oracle_prefix(w, x_cpu, T_prefix, threads):
    from oracle import oracle as O
    sl = lambda t: t[:, :T_prefix]
    t0 = time.perf_counter()
    O.gdn_fwd(sl(x_cpu["q"]), sl(x_cpu["k"]), sl(x_cpu["v"]), sl(x_cpu["a"]), sl(x_cpu["b"]),
              x_cpu["A_log"], x_cpu["dt_bias"], x_cpu["h0"], want_o=True, want_ht=True,
              threads=threads)
    return time.perf_counter() - t0


def cpu_baseline(w, x, target_s=10.0):
    """The fp64 oracle, as it stands, on the host cores: a T-prefix of the same
    workload (all heads), sized for ~target_s seconds."""
    from oracle import oracle as O
    cores = O.max_threads()
    x_cpu = {n: (t.cpu() if t is not None else None) for n, t in x.items()}
    probe_T = 64
    dt = _oracle_prefix(w, x_cpu, probe_T, cores)
    T_pre = int(min(w.T, max(probe_T, probe_T * target_s / max(dt, 1e-6))))
    T_pre = max(64, (T_pre // 64) * 64)
    dt = _oracle_prefix(w, x_cpu, T_pre, cores)
    return {"value": round(w.B * T_pre / dt, 1), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{HEADLINE} first {T_pre} of {w.T} tokens, all {w.B * w.Hv} heads, "
                      f"{dt:.1f} s wall"}


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    from oracle import oracle as O
    if rank != 0:
        return None
    w = WORKLOADS[HEADLINE]
    x = workload_inputs(w, "cpu")
    cores = O.max_threads()
    # size one step for ~3 s of wall time
    dt = _oracle_prefix(w, x, 64, cores)
    T_pre = max(64, int(min(w.T, 64 * 3.0 / max(dt, 1e-6))) // 64 * 64)
    for _ in range(args.warmup):
        _oracle_prefix(w, x, T_pre, cores)
    times = [_oracle_prefix(w, x, T_pre, cores) for _ in range(args.steps)]
    s = sum(times) / len(times)
    value = w.B * T_pre / s
    sample = f"{HEADLINE} first {T_pre} of {w.T} tokens per step, all {w.B * w.Hv} heads"
    return {"impl": "reference",
            "metric": "GDN prefill tokens/s (chunk_gated_delta_rule) on 1 B200, % of roofline",
            "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(s * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv,
                       "d": w.d, "chunk": 64},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the decode / GDN-2 / long-prefill extras")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["prefill_8k", "decode_256", "gdn2_b4_4k", "prefill_128k",
                                       "prefill_b8_16k", "conv_prefill_8k", "rmsnorm_gated_8k",
                                       "kda_b4_4k", "gate_prep_8k", "prefill_8k_gated_norm",
                                       "bwd_8k"],
                    default=None,
                    help="measure one secondary workload alone (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, local_rank, world = rank_info()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.only:
            line = run_only(args, local_rank)
        else:
            line = run_ours(args, rank, local_rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
