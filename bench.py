#!/usr/bin/env python
"""Throughput of the quantized MoE layer on B200 (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|mtp_verify|prefill|
                    mixed_prefill] [--impl ours|reference]

A step is one pass of the whole layer (a1-a7) over one batch of synthetic input:
  decode       48 independent layers (hidden 2048, 256 experts, top-8, width 512, Q4_K), one
               token each -- the default workload; one CUDA graph of 48 moe_forward calls
  mtp_verify   48 layers (hidden 2560, 512 experts, top-10 + shared, width 640), 3 tokens each
  prefill      one 4096-token chunk of the 512-expert layer (rotating over 4 layers)
  mixed_prefill one 8192-token chunk, per-expert Q4_K / Q5_K / Q8_0, Zipf(1.3) routing
The metric is MoE-layer tokens/s (tokens x layers / time); expert bytes read per step (the stored
bytes of every distinct expert that received a token, plus the shared expert) give the HBM
fraction; algorithmic int8 ops (2 * 3 * H * F per assignment) give TOPS.  The roofline object
describes the dominant kernel: for decode the fused layer kernel against HBM bandwidth (expert
bytes per launch / layer time); for prefill the gate/up grouped GEMM against the tensor-core
peak (2 * assignments * 2F * H flops per launch / its own duration, timed with CUDA events that
the library records around it in every timed step).

--impl reference times the CPU oracle (the plain fp64 C implementation under oracle/) on the
same workload, a bounded sample per step, on the host cores: the reference arm of this
comparison.  With torchrun (N > 1) every rank runs its own replica of the workload (no data
exchange: the layer needs none), timed with CUDA events and reduced as the max over ranks.
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
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; decode expert-weight GB/s and prefill int8 TOPS vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "mtp_verify", "prefill", "mixed_prefill"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: 48 decode / 4 prefill / 2 mixed_prefill); "
                         "fewer layers make a smaller case for profilers")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def traffic_for(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary (profiles/traffic.json), or None when
    that capture was of another workload or the kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("workload", "decode") != workload:
        return None
    h = hashlib.sha256()
    for s in d.get("source_files", []):
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return d["bytes_per_launch"] if d.get("source_sha256") == h.hexdigest() else None


# ------------------------------------------------------------------ ranks


def max_over_ranks(v: float, world: int, device=None) -> float:
    """The largest value over all ranks (the job's time), the same on every rank.  Every rank
    must call it at the same point (it is a collective)."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, ms: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank_step per step
    (weak scaling), the job takes ms (the max over ranks) for `steps` steps."""
    return world * units_per_rank_step * steps / (ms / 1e3)


# ------------------------------------------------------------------ workload set-up


def workload(name, layers=None):
    from expert_ffn_token_b200 import synth
    w = synth.WORKLOADS[name]
    if name in ("prefill", "mixed_prefill"):
        w = synth.with_tokens(w, w.tokens, layers=4 if name == "prefill" else 2)
    if layers is not None:
        w = synth.with_tokens(w, w.tokens, layers=layers)
    return w


def expert_bytes_and_ops(w, lay, logits):
    """Stored bytes of the distinct experts a batch touches (+ shared) and its int8 ops."""
    import numpy as np
    top = np.argsort(-logits, axis=1, kind="stable")[:, :w.k]
    used = set(int(e) for e in np.unique(top))
    if w.shared:
        used.add(w.n_experts)
    nbytes = sum(lay.expert_bytes(e) for e in used)
    assignments = logits.shape[0] * (w.k + (1 if w.shared else 0))
    ops = 2 * 3 * w.hidden * w.ffn * assignments
    return nbytes, ops, len(used)


def run_ours(args, rank, world):
    import numpy as np
    import torch

    from expert_ffn_token_b200 import moe, synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workload(args.workload, args.layers)
    decode = args.workload in ("decode", "mtp_verify")
    K = args.steps if args.steps is not None else (200 if decode else 20)
    W = args.warmup if args.warmup is not None else (10 if decode else 3)
    stream = torch.cuda.current_stream().cuda_stream

    # arenas: one tensor holding every layer, drawn on the device
    fmts0 = synth.layer_formats(w, 0)
    lays = [synth.arena_layout(w, synth.layer_formats(w, l)) for l in range(w.layers)]
    offs = [0]
    for lay in lays[:-1]:
        offs.append(offs[-1] + lay.nbytes)
    total = offs[-1] + lays[-1].nbytes
    arena = torch.empty(total, dtype=torch.uint8, device=dev)
    for l, lay in enumerate(lays):
        synth.device_fill_layer(w, l, arena.data_ptr() + offs[l], stream)
    handles = []
    for l, lay in enumerate(lays):
        handles.append(moe.arena_create(arena.data_ptr() + offs[l], lay.nbytes, w.hidden, w.ffn,
                                        w.n_experts, w.n_experts if w.shared else -1,
                                        synth.layout_descs(lay)))
    T = w.tokens
    ws_bytes = moe.workspace_size(handles[0], T, w.k, 0)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)

    # inputs (host draws, resident in HBM before timing)
    xs = np.stack([synth.activations(w, l) for l in range(w.layers)])
    lgs = np.stack([synth.router_logits(w, l) for l in range(w.layers)])
    x_d = torch.from_numpy(xs).to(dev)
    lg_d = torch.from_numpy(lgs).to(dev)
    out_d = torch.empty_like(x_d)
    step_bytes = step_ops = 0
    distinct = []
    for l in range(w.layers):
        b, o, u = expert_bytes_and_ops(w, lays[l], lgs[l])
        step_bytes += b
        step_ops += o
        distinct.append(u)
    del fmts0

    def one_step(events=None):
        for l in range(w.layers):
            if events is not None:
                moe.set_timing_events(handles[l], *[e.cuda_event for e in events[l]])
            moe.forward(handles[l], x_d[l].data_ptr(), lg_d[l].data_ptr(), T, w.k,
                        out_d[l].data_ptr(), ws.data_ptr(), ws_bytes, 0,
                        torch.cuda.current_stream().cuda_stream)

    # decode: one step (48 layers x one launch) captured in a CUDA graph.  Prefill: eager steps
    # (about ten launches per ~5 ms layer), with CUDA events around the grouped-GEMM kernels of
    # every layer of every timed step.
    graph = None
    kernels_per_step = 0
    if decode:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            one_step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        n0 = moe.kernels_enqueued()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            one_step()
        kernels_per_step = moe.kernels_enqueued() - n0
        torch.cuda.synchronize()
    step_events = []
    if not decode:
        for _ in range(K):
            row = []
            for _ in range(w.layers):
                trio = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                for e in trio:
                    e.record()          # creates the handle
                row.append(trio)
            step_events.append(row)
        torch.cuda.synchronize()

    def run(step=None):
        if graph is not None:
            graph.replay()
        else:
            one_step(step_events[step] if step is not None else None)

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    for _ in range(W):
        run()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = Clocks(os.environ.get("CUDA_VISIBLE_DEVICES", str(dev.index)).split(",")[dev.index]
                    if "CUDA_VISIBLE_DEVICES" in os.environ else dev.index)
    n0 = moe.kernels_enqueued()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        run(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if not decode:
        kernels_per_step = (moe.kernels_enqueued() - n0) // K
        for h in handles:
            moe.set_timing_events(h)
        gateup_ms = statistics.mean(t[0].elapsed_time(t[1]) for row in step_events for t in row)
        down_ms = statistics.mean(t[1].elapsed_time(t[2]) for row in step_events for t in row)
    if world > 1:
        ms = max_over_ranks(ms, world, dev)
        dist.barrier()
    clk = clocks.stop()

    # end to end through the C ABI: pinned host inputs in, result out, every step
    x_h = torch.from_numpy(xs).pin_memory()
    lg_h = torch.from_numpy(lgs).pin_memory()
    out_h = torch.empty(out_d.shape, dtype=torch.float32).pin_memory()
    for _ in range(2):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        run()
        out_h.copy_(out_d, non_blocking=True)
    torch.cuda.synchronize()
    K2 = max(3, K // 4)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(K2):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        run()
        out_h.copy_(out_d, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    ms_e2e = f0.elapsed_time(f1)
    ms_e2e = max_over_ranks(ms_e2e, world, dev)
    assert np.isfinite(out_h.numpy()).all()

    st = moe.read_status(ws.data_ptr(), stream)   # status word sits at workspace offset 0
    if st != 0:
        raise RuntimeError(f"device status {moe.status_string(st)}")
    graph = None
    for h in handles:
        moe.arena_destroy(h)

    tok_per_step = T * w.layers
    ms_step = ms / K
    hbm, bf16, src = peaks()
    if decode:
        per_launch_s = ms_step / 1e3 / w.layers
        bytes_per_launch = step_bytes / w.layers
        achieved_gbs = bytes_per_launch / per_launch_s / 1e9
        roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                    "frac": achieved_gbs / hbm,
                    "traffic": traffic_for("k_decode_fused", args.workload),
                    "kernel": "k_decode_fused (one launch per layer)",
                    "peak_source": src, "bytes_per_launch": bytes_per_launch}
    else:
        # dominant kernel: the gate/up grouped GEMM (k_gemm_tc<0>); 2 flops per multiply-add
        assign = T * (w.k + (1 if w.shared else 0))
        flops = 2.0 * assign * 2 * w.ffn * w.hidden
        achieved = flops / (gateup_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                    "frac": achieved / bf16,
                    "traffic": traffic_for("k_gemm_tc<0>", args.workload),
                    "kernel": "k_gemm_tc<0> (gate/up grouped GEMM, kind::f16 with exact integer "
                              "operands), one launch per layer",
                    "peak_source": f"{src} bf16 dense (same rate as f16)",
                    "flops_per_launch": flops, "ms_per_launch": gateup_ms,
                    "frac_of_int8_peak": achieved / (2 * bf16),
                    "down_kernel_ms_per_launch": down_ms}
    value = job_throughput(tok_per_step, K, world, ms)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": w.note, "layers": w.layers, "tokens_per_layer": T,
                   "hidden": w.hidden, "experts": w.n_experts, "top_k": w.k,
                   "shared_expert": w.shared, "ffn": w.ffn,
                   "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB of distinct expert "
                         f"bytes per step (L2 126 MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "expert_bytes_per_step": step_bytes,
        "distinct_experts_per_layer": statistics.mean(distinct),
        "expert_gbs": step_bytes / (ms_step / 1e3) / 1e9,
        "int8_tops": step_ops / (ms_step / 1e3) / 1e12,
        "roofline": roofline,
        "e2e": {"value": job_throughput(tok_per_step, K2, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": int(xs.nbytes + lgs.nbytes),
                "d2h_bytes_per_step": int(out_h.numel() * 4)},
        "gpu_launches": int(kernels_per_step * K),
        "kernels_per_step": int(kernels_per_step),
        "clocks": clk,
    }
    return result


# ------------------------------------------------------------------ oracle (CPU baseline)


def oracle_sample(w, seconds, max_layers=None):
    """Time the oracle on successive layers of the workload until ~`seconds` of CPU time."""
    import numpy as np

    import oracle
    from expert_ffn_token_b200 import synth
    oracle.build()
    threads = oracle.set_threads(0)
    done_tokens = 0
    t_total = 0.0
    layers = 0
    sample_tokens = w.tokens if w.tokens <= 64 else 16
    l = 0
    while (layers == 0 or t_total < seconds) and (max_layers is None or layers < max_layers):
        layer = l % w.layers
        x = synth.activations(w, layer)
        logits = synth.router_logits(w, layer)
        toks = np.arange(sample_tokens) if sample_tokens < w.tokens else None
        t0 = time.perf_counter()
        ids, wt, _ = oracle.topk(logits, w.k)
        t_route = time.perf_counter() - t0
        need = set(int(e) for e in ids[:sample_tokens].ravel())
        if w.shared:
            need.add(w.n_experts)
        buf, lay = synth.compact_arena(w, layer, need)       # input generation: not timed
        ex = oracle.experts_table(lay.fmts, lay.offs, lay.strides)
        t0 = time.perf_counter()
        oracle.forward(buf, ex, lay.shared, w.hidden, w.ffn, x, ids, wt, tokens=toks)
        t_total += time.perf_counter() - t0 + t_route
        done_tokens += sample_tokens
        layers += 1
        l += 1
    used = min(threads, sample_tokens)
    return {"value": done_tokens / t_total, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{layers} layer(s) x {sample_tokens} token(s) of the workload "
                      f"({t_total:.1f} s on {used} thread(s) of {host_cpu()}; OpenMP over tokens)"}


def host_cpu() -> str:
    """The host CPU's model name and the cores this process may use."""
    name = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        n = os.cpu_count() or 1
    return f"{name}, {n} usable cores"


def run_reference(args):
    w = workload(args.workload, args.layers)
    K = args.steps if args.steps is not None else 5
    W = args.warmup if args.warmup is not None else 1
    per_step = max(1.0, args.cpu_seconds / max(1, K))
    for _ in range(W):
        oracle_sample(w, 0.0, max_layers=1)
    vals = []
    t0 = time.perf_counter()
    for _ in range(K):
        vals.append(oracle_sample(w, per_step))
    wall = time.perf_counter() - t0
    v = statistics.mean(r["value"] for r in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 0, "steps": K,
            "warmup": W, "ms_per_step": 1e3 * wall / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": w.note, "layers": w.layers,
                                            "tokens_per_layer": w.tokens},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res = run_ours(args, rank, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_sample(workload(args.workload, args.layers), args.cpu_seconds)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
