#!/usr/bin/env python
"""Throughput of the quantized MoE layer on B200 (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|decode|mtp_verify|
                    prefill|mixed_prefill] [--impl ours|reference]

A step is one pass of the whole layer (a1-a7) over one batch of synthetic input of a workload:
  decode        48 independent layers (hidden 2048, 256 experts, top-8, width 512, Q4_K), one
                token each; one CUDA graph of 48 moe_forward calls -- the headline workload
  mtp_verify    48 layers (hidden 2560, 512 experts, top-10 + shared, width 640), 3 tokens each
  prefill       one 4096-token chunk of the 512-expert layer (rotating over 4 layers)
  mixed_prefill one 8192-token chunk, per-expert Q4_K / Q5_K / Q8_0, Zipf(1.3) routing
  chain         one token through 48 chained decode-shaped layers on a residual stream
                (moe_chain_forward: router in front of every layer, residual add, and the
                next layer's expert prediction prefetched into L2), one CUDA graph per step
The default (`all`) times every workload one after the other (each arena freed before the next)
and reports the decode workload as the line's headline value, the others under "workloads".
The metric is MoE-layer tokens/s (tokens x layers / time).  Per workload:
  - expert bytes read (stored bytes of every distinct expert that received a token, plus the
    shared expert) give the HBM fraction; algorithmic int8 ops (2 * 3 * H * F per assignment,
    unpadded) give TOPS; the layer's binding roofline is max(bytes / HBM, ops / int8 peak);
  - `roofline` describes the dominant kernel: decode -- the fused layer kernel against HBM
    bandwidth (expert bytes per launch / layer time); prefill -- the gate/up grouped GEMM against
    the fp16 tensor-core peak (2 * assignments * 2F * H flops per launch / its own duration, from
    CUDA events the library records around it in every timed step);
  - `e2e` goes through the C ABI eagerly (moe_forward per layer) with the inputs copied from
    pinned host memory and the outputs copied back inside the timed region;
  - `cpu_baseline` is the plain fp64 C oracle (oracle/) timed on the host's cores on a bounded
    sample of the same workload, all cores and one thread.

--impl reference times that oracle alone on the headline workload (the reference arm).  With
torchrun (N > 1) every rank runs its own replica of the workloads (no data exchange: the layer
needs none), timed with CUDA events and reduced as the max over ranks.
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
INT8_NOMINAL_TOPS = 4500.0          # B200 dense int8, datasheet figure
ALL = ("decode", "mtp_verify", "prefill", "mixed_prefill", "chain")
HEADLINE = "decode"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="all", choices=["all", *ALL])
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="target CPU time of each oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: 48 decode / 4 prefill / 2 mixed_prefill); "
                         "fewer layers make a smaller case for profilers")
    return ap.parse_args(argv)


def peaks():
    """(HBM GB/s, bf16 dense TFLOP/s, source): the driver's measured figures, else fallback."""
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
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        """Rows sampled so far: [(sm_mhz, max_mhz, reasons set)]."""
        if self.p is None:
            return None
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        out = []
        for r in rows:
            try:
                out.append((float(r[1]), float(r[2]),
                            {self.NAMES[i] for i in range(4) if r[5 + i].strip() == "Active"}))
            except ValueError:
                pass
        return out

    @staticmethod
    def summary(rows):
        if rows is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(set().union(*(r[2] for r in rows))), "samples": len(rows)}


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json), or None when
    that capture was of another workload or the kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        table = json.load(f)
    d = table.get(f"{kernel}@{workload}")
    if not d:
        return None
    h = hashlib.sha256()
    try:
        for s in d.get("source_files", []):
            with open(os.path.join(ROOT, s), "rb") as f:
                h.update(f.read())
    except OSError:           # a source of that capture no longer exists
        return None
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


def run_workload(name, args, world, dev):
    """Time one workload on this rank's GPU; returns its result dict (every rank, same keys)."""
    import numpy as np
    import torch

    from expert_ffn_token_b200 import moe, synth

    w = workload(name, args.layers)
    decode = name in ("decode", "mtp_verify")
    K = args.steps if args.steps is not None else (200 if decode else 20)
    W = args.warmup if args.warmup is not None else (10 if decode else 3)
    stream = torch.cuda.current_stream().cuda_stream

    # arenas: one tensor holding every layer, drawn on the device
    lays = [synth.arena_layout(w, synth.layer_formats(w, l)) for l in range(w.layers)]
    offs = [0]
    for lay in lays[:-1]:
        offs.append(offs[-1] + lay.nbytes)
    total = offs[-1] + lays[-1].nbytes
    arena = torch.empty(total, dtype=torch.uint8, device=dev)
    for l in range(w.layers):
        synth.device_fill_layer(w, l, arena.data_ptr() + offs[l], stream)
    handles = [moe.arena_create(arena.data_ptr() + offs[l], lay.nbytes, w.hidden, w.ffn,
                                w.n_experts, w.n_experts if w.shared else -1,
                                synth.layout_descs(lay)) for l, lay in enumerate(lays)]
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

    # prefill: the gate/up phase on kind::i8 products (the default) or on exact kind::f16
    # products (timed beside it)
    main_flags = 0 if decode else moe.F_TC_I8

    def one_step(events=None, flags=None):
        fl = main_flags if flags is None else flags
        for l in range(w.layers):
            if events is not None:
                moe.set_timing_events(handles[l], *[e.cuda_event for e in events[l]])
            moe.forward(handles[l], x_d[l].data_ptr(), lg_d[l].data_ptr(), T, w.k,
                        out_d[l].data_ptr(), ws.data_ptr(), ws_bytes, fl,
                        torch.cuda.current_stream().cuda_stream)

    # decode: one step (the layers' single launches) captured in a CUDA graph.  Prefill: eager
    # steps (about ten launches per layer) with CUDA events around the grouped-GEMM kernels of
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
    gpu_id = (os.environ["CUDA_VISIBLE_DEVICES"].split(",")[dev.index]
              if "CUDA_VISIBLE_DEVICES" in os.environ else dev.index)
    clocks = Clocks(gpu_id)
    n0 = moe.kernels_enqueued()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        run(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    gateup_ms = down_ms = None
    if not decode:
        kernels_per_step = (moe.kernels_enqueued() - n0) // K
        for h in handles:
            moe.set_timing_events(h)
        gateup_ms = statistics.mean(t[0].elapsed_time(t[1]) for row in step_events for t in row)
        down_ms = statistics.mean(t[1].elapsed_time(t[2]) for row in step_events for t in row)
    ms = max_over_ranks(ms, world, dev)
    if world > 1:
        dist.barrier()
    clock_rows = clocks.stop()

    # prefill: the other gate/up kernel on the same inputs, same steps (its own warm-up)
    alt = None
    if not decode:
        for _ in range(W):
            one_step(flags=0)
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for i in range(K):
            one_step(step_events[i], flags=0)
        g1.record()
        torch.cuda.synchronize()
        for h in handles:
            moe.set_timing_events(h)
        alt = {"ms": max_over_ranks(g0.elapsed_time(g1), world, dev),
               "gateup_ms": statistics.mean(t[0].elapsed_time(t[1])
                                            for row in step_events for t in row),
               "down_ms": statistics.mean(t[1].elapsed_time(t[2])
                                          for row in step_events for t in row)}

    # end to end through the C ABI, eagerly: pinned host inputs in, every layer's moe_forward,
    # the result out, every step
    x_h = torch.from_numpy(xs).pin_memory()
    lg_h = torch.from_numpy(lgs).pin_memory()
    out_h = torch.empty(out_d.shape, dtype=torch.float32).pin_memory()

    def e2e_step(graphed):
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        if graphed:
            graph.replay()
        else:
            one_step()
        out_h.copy_(out_d, non_blocking=True)

    def time_e2e(graphed):
        for _ in range(2):
            e2e_step(graphed)
        torch.cuda.synchronize()
        k2 = max(3, K // 4)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(k2):
            e2e_step(graphed)
        f1.record()
        torch.cuda.synchronize()
        return k2, max_over_ranks(f0.elapsed_time(f1), world, dev)

    k2, ms_e2e = time_e2e(False)
    graph_e2e = time_e2e(True) if graph is not None else None
    assert np.isfinite(out_h.numpy()).all()

    st = moe.read_status(ws.data_ptr(), stream)   # status word sits at workspace offset 0
    if st != 0:
        raise RuntimeError(f"{name}: device status {moe.status_string(st)}")
    graph = None
    for h in handles:
        moe.arena_destroy(h)
    del arena, ws, x_d, lg_d, out_d
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    tok_per_step = T * w.layers
    ms_step = ms / K
    layer_s = ms_step / 1e3 / w.layers
    hbm, bf16, src = peaks()
    bytes_per_layer = step_bytes / w.layers
    ops_per_layer = step_ops / w.layers
    int8_meas = 2.0 * bf16           # the int8 tensor rate is twice the fp16/bf16 rate
    t_hbm = bytes_per_layer / (hbm * 1e9)
    t_tensor = ops_per_layer / (int8_meas * 1e12)
    layer_roof = {"t_min_us": 1e6 * max(t_hbm, t_tensor),
                  "binding": "hbm" if t_hbm >= t_tensor else "int8 tensor",
                  "t_hbm_us": 1e6 * t_hbm, "t_int8_us": 1e6 * t_tensor,
                  "frac": max(t_hbm, t_tensor) / layer_s,
                  "int8_peak_tops": int8_meas,
                  "int8_peak_source": f"2 x {src} bf16 dense ({bf16:.1f} TFLOP/s)"}
    if decode:
        achieved = bytes_per_layer / layer_s / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "traffic": traffic_for("k_decode_fused", name),
                    "kernel": "k_decode_fused (one launch per layer)",
                    "peak_source": f"{src} HBM copy", "bytes_per_launch": bytes_per_layer}
    else:
        # dominant kernel: the gate/up grouped GEMM on int8 products (k_gateup_i8), against the
        # int8 dense peak; 2 ops per multiply-add
        assign = T * (w.k + (1 if w.shared else 0))
        flops = 2.0 * assign * 2 * w.ffn * w.hidden
        achieved = flops / (gateup_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": int8_meas, "unit": "TOP/s",
                    "frac": achieved / int8_meas, "traffic": traffic_for("k_gateup_i8", name),
                    "kernel": "k_gateup_i8 (gate/up grouped GEMM, tcgen05 kind::i8: one s32 "
                              "accumulator per 32-weight block, promoted in fp32), one launch "
                              "per layer",
                    "peak_source": f"int8 dense = 2 x {src} bf16 dense ({bf16:.1f} TFLOP/s)",
                    "ops_per_launch": flops, "ms_per_launch": gateup_ms,
                    "frac_of_bf16_peak": achieved / bf16,
                    "down_ms_per_launch": down_ms,
                    "down_note": "k_h_rows + k_down_tc, from the events around the down phase"}
        f16_ach = flops / (alt["gateup_ms"] / 1e3) / 1e12
        alt_layer_s = alt["ms"] / K / 1e3 / w.layers
        roofline["f16_variant"] = {
            "kernel": "k_gateup_tc (tcgen05 kind::f16: exact integer weight operands, hi/lo "
                      "activation planes), timed on the same inputs after the main loop",
            "ms_per_launch": alt["gateup_ms"], "achieved_tflops": f16_ach,
            "frac_of_bf16_peak": f16_ach / bf16, "frac_of_int8_peak": f16_ach / int8_meas,
            "traffic": traffic_for("k_gateup_tc", name),
            "down_ms_per_launch": alt["down_ms"], "us_per_layer": 1e6 * alt_layer_s,
            "value": job_throughput(T * w.layers, K, world, alt["ms"]), "unit": "tokens/s"}
    res = {
        "workload": w.note, "value": job_throughput(tok_per_step, K, world, ms),
        "unit": "tokens/s", "steps": K, "warmup": W, "ms_per_step": ms_step,
        "us_per_layer": 1e6 * layer_s, "layers": w.layers, "tokens_per_layer": T,
        "hidden": w.hidden, "experts": w.n_experts, "top_k": w.k, "shared_expert": w.shared,
        "ffn": w.ffn,
        "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB of distinct expert bytes per "
              f"step (L2 126 MB)",
        "expert_bytes_per_step": step_bytes,
        "distinct_experts_per_layer": statistics.mean(distinct),
        "expert_gbs": step_bytes / (ms_step / 1e3) / 1e9,
        "int8_tops": step_ops / (ms_step / 1e3) / 1e12,
        "int8_frac_of_nominal": step_ops / (ms_step / 1e3) / 1e12 / INT8_NOMINAL_TOPS,
        "layer_roofline": layer_roof,
        "roofline": roofline,
        "e2e": {"value": job_throughput(tok_per_step, k2, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": int(xs.nbytes + lgs.nbytes),
                "d2h_bytes_per_step": int(out_h.numel() * 4),
                "mode": "eager moe_forward per layer through the C ABI"},
        "gpu_launches": int(kernels_per_step * K),
        "kernels_per_step": int(kernels_per_step),
        "clock_rows": clock_rows,
    }
    if graph_e2e is not None:
        res["e2e_graph"] = {"value": job_throughput(tok_per_step, graph_e2e[0], world,
                                                    graph_e2e[1]),
                            "unit": "tokens/s", "mode": "the captured graph of moe_forward calls"}
    return res


def run_chain(name, args, world, dev):
    """One token through 48 chained decode-shaped layers (moe_chain_forward with the lookahead),
    one CUDA graph per step; the same chain without the lookahead timed beside it."""
    import numpy as np
    import torch

    from expert_ffn_token_b200 import moe, synth

    w = workload("decode", args.layers)
    K = args.steps if args.steps is not None else 50
    W = args.warmup if args.warmup is not None else 5
    stream = torch.cuda.current_stream().cuda_stream
    lays = [synth.arena_layout(w, synth.layer_formats(w, l)) for l in range(w.layers)]
    offs = [0]
    for lay in lays[:-1]:
        offs.append(offs[-1] + lay.nbytes)
    arena = torch.empty(offs[-1] + lays[-1].nbytes, dtype=torch.uint8, device=dev)
    for l in range(w.layers):
        synth.device_fill_layer(w, l, arena.data_ptr() + offs[l], stream)
    handles = [moe.arena_create(arena.data_ptr() + offs[l], lay.nbytes, w.hidden, w.ffn,
                                w.n_experts, -1, synth.layout_descs(lay))
               for l, lay in enumerate(lays)]
    # router rows: N(0, 0.05^2) fp32, drawn on the device from a seeded generator
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    routers = torch.randn((w.layers, w.n_experts, w.hidden), generator=gen, device=dev) * 0.05
    # RMSNorm weight 1/32: keeps the random (not zero-mean) experts' h inside the fp16 range of
    # its Q8_1 scales along the chain
    gamma = torch.full((w.hidden,), 2.0 ** -5, dtype=torch.float32, device=dev)
    layers = [(handles[l], routers[l].data_ptr(), None, gamma.data_ptr())
              for l in range(w.layers)]
    T, k, H = w.tokens, w.k, w.hidden
    x0 = synth.activations(w, 0)
    x_d = torch.from_numpy(x0).to(dev)
    xo_d = torch.empty_like(x_d)
    fl_on, fl_off = moe.F_LOOKAHEAD, 0
    ws_bytes = moe.chain_workspace_size(layers, T, k, fl_on)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)

    # one traced run: the ids of every layer (expert bytes per step) and the lookahead's hits
    ids_t = torch.empty((w.layers, T, k), dtype=torch.int32, device=dev)
    early_t = torch.full((w.layers, T, k), -1, dtype=torch.int32, device=dev)
    moe.chain_forward(layers, x_d.data_ptr(), T, k, xo_d.data_ptr(), ws.data_ptr(), ws_bytes,
                      fl_on, {"ids": ids_t.data_ptr(), "early": early_t.data_ptr()}, stream)
    torch.cuda.synchronize()
    ids = ids_t.cpu().numpy()
    early = early_t.cpu().numpy()
    hits = sum(len(set(ids[l].ravel()) & set(early[l].ravel())) for l in range(1, w.layers))
    picks = sum(len(set(ids[l].ravel())) for l in range(1, w.layers))
    step_bytes = sum(sum(lays[l].expert_bytes(int(e)) for e in set(ids[l].ravel()))
                     for l in range(w.layers))

    def capture(flags):
        def one():
            moe.chain_forward(layers, x_d.data_ptr(), T, k, xo_d.data_ptr(), ws.data_ptr(),
                              ws_bytes, flags, None, torch.cuda.current_stream().cuda_stream)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            one()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        n0 = moe.kernels_enqueued()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one()
        n = moe.kernels_enqueued() - n0
        torch.cuda.synchronize()
        return g, n, one

    g_on, kern_on, eager_on = capture(fl_on)
    g_off, _, _ = capture(fl_off)

    def timed(fn, steps):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    gpu_id = (os.environ["CUDA_VISIBLE_DEVICES"].split(",")[dev.index]
              if "CUDA_VISIBLE_DEVICES" in os.environ else dev.index)
    clocks = Clocks(gpu_id)
    ms = timed(g_on.replay, K)
    ms_off = timed(g_off.replay, K)
    clock_rows = clocks.stop()

    # end to end through the C ABI: x0 from pinned host memory, moe_chain_forward (eager), x_L
    # back to the host, every step
    x_h = torch.from_numpy(x0).pin_memory()
    xo_h = torch.empty(xo_d.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        eager_on()
        xo_h.copy_(xo_d, non_blocking=True)

    k2 = max(3, K // 2)
    ms_e2e = timed(e2e_step, k2)
    assert np.isfinite(xo_h.numpy()).all()
    st = moe.read_status(moe.chain_status_word(layers, ws.data_ptr(), T, k, fl_on), stream)
    if st != 0:
        raise RuntimeError(f"chain: device status {moe.status_string(st)}")
    sample = {"w": w, "x0": x0, "ids": ids, "routers": routers.cpu().numpy(),
              "norm": gamma.cpu().numpy()}
    g_on = g_off = None
    for h in handles:
        moe.arena_destroy(h)
    del arena, ws, routers
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    hbm, _, src = peaks()
    ms_step = ms / K
    layer_s = ms_step / 1e3 / w.layers
    achieved = step_bytes / w.layers / layer_s / 1e9
    return {
        "workload": "one token through 48 chained decode-shaped layers (hidden 2048, 256 "
                    "experts, top-8, width 512, Q4_K) on a residual stream: RMSNorm (weight "
                    "1/32) + router (fp32 rows N(0, 0.05^2)) + layer + residual add per layer, "
                    "lookahead prefetch on",
        "value": job_throughput(T * w.layers, K, world, ms), "unit": "tokens/s",
        "steps": K, "warmup": W, "ms_per_step": ms_step, "us_per_layer": 1e6 * layer_s,
        "layers": w.layers, "tokens_per_layer": T, "hidden": H, "experts": w.n_experts,
        "top_k": k, "shared_expert": False, "ffn": w.ffn,
        "chain_tokens_per_s": job_throughput(T, K, world, ms),
        "lookahead_off": {"ms_per_step": ms_off / K,
                          "us_per_layer": 1e3 * ms_off / K / w.layers,
                          "value": job_throughput(T * w.layers, K, world, ms_off)},
        "lookahead_hit_rate": hits / max(1, picks),
        "l2": f"{step_bytes / 1e6:.0f} MB of distinct expert bytes per step (L2 126 MB)",
        "expert_bytes_per_step": step_bytes,
        "expert_gbs": step_bytes / (ms_step / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None,
                     "kernel": "the chained layer (k_router_rows + k_decode_fused per layer): "
                               "expert bytes per layer / layer time",
                     "peak_source": f"{src} HBM copy"},
        "e2e": {"value": job_throughput(T * w.layers, k2, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x0.nbytes), "d2h_bytes_per_step": int(xo_h.numel() * 4),
                "mode": "eager moe_chain_forward through the C ABI"},
        "gpu_launches": int(kern_on * K),
        "kernels_per_step": int(kern_on),
        "clock_rows": clock_rows,
        "_chain_sample": sample,
    }


# ------------------------------------------------------------------ oracle (CPU baseline)


def chain_oracle_sample(cs, seconds, threads=None):
    """The oracle's chain (O10, O3, O1-O9 and the residual add per layer) on the first layers of
    the chain workload, from the same x0 and router rows, until ~`seconds` of CPU time.  The
    arenas hold the experts the GPU's chain chose (input generation, not timed); a layer whose
    oracle ids differ from them ends the sample (its arena would lack those experts)."""
    import numpy as np

    import oracle
    from expert_ffn_token_b200 import synth
    oracle.build()
    used = oracle.set_threads(threads if threads else host_cores())
    w = cs["w"]
    x = cs["x0"]
    t_total, layers, l = 0.0, 0, 0
    while layers == 0 or t_total < seconds:
        if l == len(cs["routers"]):     # the whole chain done: start again from x0
            l, x = 0, cs["x0"]
        buf, lay = synth.compact_arena(w, l, set(int(e) for e in cs["ids"][l].ravel()))
        L = {"arena": buf, "experts": oracle.experts_table(lay.fmts, lay.offs, lay.strides),
             "shared": -1, "hidden": w.hidden, "ffn": w.ffn, "router": cs["routers"][l],
             "norm": cs["norm"]}
        t0 = time.perf_counter()
        x_next, ids = oracle.chain([L], x, w.k)
        t_total += time.perf_counter() - t0
        layers += 1
        if not np.array_equal(ids[0], cs["ids"][l]):
            break
        x = x_next
        l += 1
    return {"value": layers * w.tokens / t_total, "unit": "tokens/s", "cores": used,
            "kind": "oracle",
            "sample": f"{layers} chained layer(s) x {w.tokens} token(s) (router, top-k, layer, "
                      f"residual); {t_total:.1f} s on {used} thread(s) of {host_cpu()}"}



def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_sample(w, seconds, max_layers=None, threads=None):
    """Time the oracle on successive layers of the workload until ~`seconds` of CPU time, on
    `threads` OpenMP threads (default: every usable core)."""
    import numpy as np

    import oracle
    from expert_ffn_token_b200 import synth
    oracle.build()
    used = oracle.set_threads(threads if threads else host_cores())
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
    what = "all tokens" if sample_tokens == w.tokens else f"{sample_tokens} of {w.tokens} tokens"
    return {"value": done_tokens / t_total, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{layers} layer(s) x {sample_tokens} token(s) of the workload ({what} "
                      f"per layer; {t_total:.1f} s on {used} thread(s) of {host_cpu()}; OpenMP "
                      f"over the rows of each expert matrix)"}


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
    return f"{name}, {host_cores()} usable cores"


def run_reference(args):
    name = HEADLINE if args.workload == "all" else args.workload
    w = workload(name, args.layers)
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
    import torch
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    names = ALL if args.workload == "all" else (args.workload,)
    results = {n: (run_chain if n == "chain" else run_workload)(n, args, world, dev)
               for n in names}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for n in names:
            if n == "chain":
                cs = results[n].pop("_chain_sample")
                results[n]["cpu_baseline"] = chain_oracle_sample(cs, args.cpu_seconds)
                results[n]["cpu_baseline_1_thread"] = chain_oracle_sample(cs, args.cpu_seconds / 2,
                                                                          threads=1)
                continue
            w = workload(n, args.layers)
            results[n]["cpu_baseline"] = oracle_sample(w, args.cpu_seconds)
            results[n]["cpu_baseline_1_thread"] = oracle_sample(w, args.cpu_seconds / 2,
                                                                threads=1)
    for r in results.values():
        r.pop("_chain_sample", None)
    head_name = HEADLINE if HEADLINE in results else names[0]
    all_rows = []
    for r in results.values():
        rows = r.pop("clock_rows")
        r["clocks"] = Clocks.summary(rows)
        all_rows.extend(rows or [])
    head = results[head_name]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": head["steps"], "warmup": head["warmup"], "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded generator; random-init Q4_K/Q5_K/Q8_0 experts)",
        "config": {"workload": head["workload"], "layers": head["layers"],
                   "tokens_per_layer": head["tokens_per_layer"], "hidden": head["hidden"],
                   "experts": head["experts"], "top_k": head["top_k"],
                   "shared_expert": head["shared_expert"], "ffn": head["ffn"],
                   "l2": head["l2"],
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "expert_gbs": head["expert_gbs"], "int8_tops": head.get("int8_tops"),
        "roofline": head["roofline"], "layer_roofline": head.get("layer_roofline"),
        "e2e": head["e2e"],
        "gpu_launches": sum(r["gpu_launches"] for r in results.values()),
        "clocks": Clocks.summary(all_rows if all_rows else None),
        "workloads": results,
    }
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
