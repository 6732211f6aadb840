#!/usr/bin/env python
"""Benchmark of the cascade-pruned attention path (SpAtten-style) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one spatten_cascade_forward over the BERT-base-shaped prefill workload: B=32
sequences of T=512 tokens, d_model 768, 12 heads of 64, 12 layers, token keep 0.9 per layer,
one head dropped every 3 layers, 12-bit progressive K/V (8-bit MSB + 4-bit LSB planes), refetch
when a row's max probability < 0.1, 5 % of tokens with K rows x4.  Inputs are seeded synthetic
draws with random-init weights (bf16), resident in HBM before the timed region.  Metric: tokens/s
(B*T per step, summed over ranks; weak scaling: each rank runs its own batch, no collective on the
data path).  L2 is flushed (a 256 MB write) between timed steps, outside the timed events.

The JSON line also carries the roofline of the attention kernel (timed live per layer with CUDA
events recorded around its launches on the launching stream), the end-to-end rate through the C
ABI with host buffers (H2D of the inputs and D2H of the results inside the timed region), SM
clocks sampled during the timed region, and the float64 CPU oracle timed on a bounded sample.
`--impl reference` times that oracle alone, as the reference arm.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def attention_flops(w) -> float:
    """Algorithmic attention flops of one prefill step: 4 * k_l^2 * d_h per kept head and sequence
    (Q K^T and P V on the kept tokens)."""
    return float(sum(w.B * w.head_keep[l] * 4.0 * w.token_keep[l] ** 2 * w.d_h for l in range(w.L)))


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.tmp.read().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.tmp.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ------------------------------------------------------------------------------------------------
def oracle_sample(w, d, seconds: float, max_seqs: int | None = None):
    """Run the float64 oracle cascade one sequence at a time until `seconds` elapsed (at least one
    sequence).  Returns (tokens/s, sequences done, wall seconds, threads)."""
    import numpy as np
    import torch
    from oracle import spatten_ref as R

    def cast(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()

    wq = [cast(a) for a in d["w_qkv"]]
    wo = [cast(a) for a in d["w_o"]]
    done, t0 = 0, time.perf_counter()
    while True:
        b = done % w.B
        X = cast(d["X"][b:b + 1])
        g = None if d["key_gain"] is None else d["key_gain"][b:b + 1]
        R.cascade_prefill(X, wq, wo, w.H, w.d_h, w.token_keep, w.head_keep, w.quant, w.theta, key_gain=g)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_seqs and done >= max_seqs):
            break
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    return done * w.T / el, done, el, threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from cascade_token_head_b200 import synth
    w = synth.bert_base_prefill()
    d = synth.draw_prefill(w)
    for _ in range(args.warmup):
        oracle_sample(w, d, 0.0, max_seqs=1)
    t0 = time.perf_counter()
    threads = 1
    for _ in range(args.steps):
        _, _, _, threads = oracle_sample(w, d, 0.0, max_seqs=1)
    el = time.perf_counter() - t0
    value = args.steps * w.T / el
    line = {"metric": "pruned-attn tokens/s (BERT-base prefill, cascade token/head pruning, progressive K/V)",
            "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded N(0,1) activations, random-init weights)",
            "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.T, "parallelism": "replicas"},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"one sequence (T={w.T}, all {w.L} layers) of the workload per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from cascade_token_head_b200 import spatten as S
    from cascade_token_head_b200 import synth

    w = synth.bert_base_prefill()
    w.seed = rank
    d = synth.draw_prefill(w)
    bf = torch.bfloat16
    B, T, D, H, L = w.B, w.T, w.D, w.H, w.L
    X_host = torch.from_numpy(d["X"]).to(bf).pin_memory()
    gain_host = torch.from_numpy(d["key_gain"].astype(np.float32)).pin_memory()
    X = X_host.to(dev)
    gain = gain_host.to(dev)
    W = [(torch.from_numpy(d["w_qkv"][l]).to(bf).to(dev), torch.from_numpy(d["w_o"][l]).to(bf).to(dev))
         for l in range(L)]
    kl = w.token_keep[-1]
    x_out = torch.empty((B, kl, D), dtype=bf, device=dev)
    kept_tok = torch.empty((L, B, T), dtype=torch.int32, device=dev)
    kept_head = torch.empty((L, B, H), dtype=torch.int32, device=dev)
    tok_imp = torch.empty((B, T), dtype=torch.float32, device=dev)
    head_imp = torch.empty((B, H), dtype=torch.float32, device=dev)
    refetch = torch.empty(L, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cfg = S.make_cfg(S.PREFILL, B, T, D, H, w.d_h, L, S.BF16, w.token_keep, w.head_keep, True, w.theta)
    ws = torch.empty(S.cascade_workspace_size(cfg), dtype=torch.uint8, device=dev)
    io = S.cascade_io()
    io.x, io.key_gain, io.x_out = X.data_ptr(), gain.data_ptr(), x_out.data_ptr()
    io.kept_tok, io.kept_head = kept_tok.data_ptr(), kept_head.data_ptr()
    io.tok_imp, io.head_imp, io.refetch_count = tok_imp.data_ptr(), head_imp.data_ptr(), refetch.data_ptr()
    io.dev_status = status.data_ptr()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        S.cascade_forward(cfg, W, io, ws, ws.numel(), stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status after warm-up"

    # per-step events and per-layer attention-kernel events (recorded by the library inside the
    # captured step); the step is captured once into a CUDA graph and replayed K times
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    attn_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * L)]
    for e in attn_ev:      # materialise the CUDA events before handing their handles over
        e.record(stream)
    torch.cuda.synchronize()
    import ctypes as C
    attn_array = (C.c_void_p * (2 * L))(*[e.cuda_event for e in attn_ev])
    io.attn_events = C.cast(attn_array, C.POINTER(C.c_void_p))
    graph = None
    launches_per_step = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        l0 = S.kernel_launch_count()
        with torch.cuda.graph(graph):
            S.cascade_forward(cfg, W, io, ws, ws.numel(), stream=torch.cuda.current_stream())
        launches_per_step = S.kernel_launch_count() - l0
        graph.replay()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = S.kernel_launch_count()
    clocks.start()
    time.sleep(0.3)
    attn_ms = []
    for i in range(K):
        flush.zero_()
        ev_s[i].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        ev_e[i].record(stream)
        torch.cuda.synchronize()   # read this step's attention events before the next replay
        attn_ms.append(sum(attn_ev[2 * l].elapsed_time(attn_ev[2 * l + 1]) for l in range(L)))
    torch.cuda.synchronize()
    clk = clocks.stop()
    launches = (launches_per_step * K) if graph is not None else S.kernel_launch_count() - launches0
    if world > 1:
        dist.barrier()
    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(K)]
    io.attn_events = None
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    assert int(status.item()) == 0, "device status after timing"
    refetch_rows = refetch.cpu().tolist()

    # end to end through the C ABI with host buffers: H2D of X and key_gain, forward, D2H of the
    # final rows, the kept sets and the cumulative importance
    out_host = torch.empty_like(x_out, device="cpu").pin_memory()
    kept_host = torch.empty_like(kept_tok, device="cpu").pin_memory()
    imp_host = torch.empty_like(tok_imp, device="cpu").pin_memory()
    h2d = X_host.numel() * X_host.element_size() + gain_host.numel() * 4
    d2h = out_host.numel() * 2 + kept_host.numel() * 4 + imp_host.numel() * 4
    e2e_ms = []
    for i in range(max(3, K // 2)):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        X.copy_(X_host, non_blocking=True)
        gain.copy_(gain_host, non_blocking=True)
        step()
        out_host.copy_(x_out, non_blocking=True)
        kept_host.copy_(kept_tok, non_blocking=True)
        imp_host.copy_(tok_imp, non_blocking=True)
        b_.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(a.elapsed_time(b_))
    e2e_total = sum(e2e_ms)
    if world > 1:
        t = torch.tensor([e2e_total], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total = float(t.item())

    tokens_per_step = B * T
    value = world * tokens_per_step * K / (total_ms / 1e3)
    e2e_value = world * tokens_per_step * len(e2e_ms) / (e2e_total / 1e3)
    peaks, peak_kind = load_peaks()
    flops = attention_flops(w)
    attn_s = statistics.mean(attn_ms) / 1e3
    achieved = flops / attn_s / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))

    result = {
        "metric": "pruned-attn tokens/s (BERT-base prefill, cascade token/head pruning, progressive K/V)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) activations, random-init weights)",
        "config": {"workload": w.name, "global_batch": B * world, "seq_len": T, "d_model": D, "heads": H,
                   "layers": L, "token_keep": w.token_keep, "head_keep": w.head_keep, "refetch_threshold": w.theta,
                   "parallelism": f"dp{world} (independent sequences)", "l2": "flushed between timed steps",
                   "launch": "CUDA graph of one step" if graph is not None else "direct launches"},
        "roofline": {"kernel": "attention (spatten_attention_layer main kernel, all layers)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 sustained", "traffic": None,
                     "algorithmic_flops_per_step": flops, "attn_ms_per_step": attn_s * 1e3},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "clocks": clk,
        "refetch_rows_per_layer": refetch_rows,
    }
    if rank == 0 and not args.no_cpu_baseline:
        v, n, el, threads = oracle_sample(w, d, args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                  "sample": f"{n} sequence(s) of the workload (T={T}, all {L} layers), {el:.1f} s"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the step directly instead of replaying a CUDA graph")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    raise SystemExit(main())
