#!/usr/bin/env python
"""Benchmark of the cascade-pruned attention path (SpAtten-style) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload bert_base_prefill|gpt2m_decode|long_prefill]

Default (one JSON line): the BERT-base-shaped prefill, with the GPT-2-medium-shaped decode in the
line's "decode" object.
* Prefill step: one spatten_cascade_forward over B=32 sequences of T=512 tokens, d_model 768, 12
  heads of 64, 12 layers, token keep 0.9 per layer, one head dropped every 3 layers, 12-bit
  progressive K/V (8-bit MSB + 4-bit LSB planes), refetch when a row's max probability < 0.1, 5 %
  of tokens with K rows x4.  tokens/s = B*T per step.
* Decode step: one generation of 128 tokens for B=16 sequences after a 1024-token prompt (24
  layers, 16 heads of 64, d_model 1024), the K/V caches quantized once before timing, the cache
  pruned by cumulative importance to 50 % by the last layer, refetch below 0.2.  One
  spatten_cascade_forward per generated token.  tokens/s = B*128 per step.
* long_prefill: B=1, T=16384, d_model 4096, 32 heads of 128, 4 layers, keep 0.5 per layer.
Inputs are seeded synthetic draws with random-init weights (bf16), resident in HBM before the timed
region; each timed step is one CUDA-graph replay; L2 is flushed (a 256 MB write) between timed
steps, outside the timed events.  Weak scaling: each rank runs its own sequences, no collective
on the data path; the value sums all ranks over the slowest rank's time.

Each line carries the roofline of the dominant kernel (attention; timed live with CUDA events
recorded by the library around its launches on the launching stream), the end-to-end rate through
the C ABI with host buffers (H2D of the inputs and D2H of the results inside the timed region), SM
clocks sampled during the timed region, and the float64 CPU oracle timed on a bounded sample.
`--impl reference` times that oracle alone, as the reference arm.
"""
from __future__ import annotations

import argparse
import ctypes as C
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
METRIC = {
    "bert_base_prefill": "pruned-attn tokens/s (BERT-base prefill, cascade token/head pruning, progressive K/V)",
    "long_prefill": "pruned-attn tokens/s (long-context prefill, cascade token/head pruning, progressive K/V)",
    "gpt2m_decode": "generated tokens/s (GPT-2-medium decode, cumulative cache pruning, progressive K/V)",
}
DATA = "synthetic (seeded N(0,1) activations, random-init weights)"


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the prefill attention kernels of
# one BERT-base-shaped layer (32 sequences, 12 heads of 64, 512 keys, refetch below 0.1), summed
# over attn_main, attn_full and attn_reduce from one ncu capture of
#   python -m cascade_token_head_b200.cases attention --B 32 --H 12 --n 512 --d 64 --theta 0.1 --reps 1
# with --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum -k regex:attn_ -c 3.
# The capture belongs to the sources whose hash it carries: once any of them changes the line
# reports traffic null until the kernels are captured again.
TRAFFIC_SOURCES = ("attn_tc.cu", "attn_reduce.cu", "tc_ptx.cuh", "exp2_poly.cuh", "common.cuh")
CAPTURED_TRAFFIC = {
    "prefill_attention_layer": {"sources_sha256": "48619f953440a3a2", "bytes": 50435328 + 1255168 + 39167232 + 4048640,
                                "kept_key_heads": 512 * 12},
}


def sources_hash(files=TRAFFIC_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "cascade_token_head_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def prefill_traffic(w):
    """DRAM bytes of one step's attention launches: the captured layer scaled by the step's
    sum over layers of kept keys x kept heads (null when the kernels changed since the capture)."""
    c = CAPTURED_TRAFFIC["prefill_attention_layer"]
    if w.name != "bert_base_prefill_bf16":
        return None, "null: no DRAM capture of this workload's layer shape"
    try:
        current = sources_hash()
    except OSError:
        return None, "null: the kernel sources are not beside this package"
    if current != c["sources_sha256"]:
        return None, "null: the attention kernels changed since their DRAM capture"
    units = sum(w.token_keep[l] * w.head_keep[l] for l in range(w.L))
    per_seq = c["bytes"] / 32.0
    return per_seq * w.B * units / c["kept_key_heads"], (
        "ncu capture of one 32x12x512 layer (attn_main + attn_full + attn_reduce), scaled by the step's "
        "sum over layers of kept keys x kept heads and by the batch")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def prefill_workload(name):
    from cascade_token_head_b200 import synth
    return {"bert_base_prefill": synth.bert_base_prefill, "long_prefill": synth.long_prefill}[name]()


def attention_flops(w) -> float:
    """Algorithmic attention flops of one prefill step: 4 * k_l^2 * d_h per kept head and sequence
    (Q K^T and P V on the kept tokens)."""
    return float(sum(w.B * w.head_keep[l] * 4.0 * w.token_keep[l] ** 2 * w.d_h for l in range(w.L)))


def decode_attention_bytes(w, refetch_rows) -> float:
    """Algorithmic bytes of the decode attention launches of one generation: per layer and token,
    the MSB planes of K and V of the kept rows (B*H*k*d_h*2), the packed LSB planes of K and V for
    every refetched (sequence, head) row (k*d_h), and the kept-row index list (B*k*4).
    refetch_rows[s][l]: refetched (sequence, head) rows of token s, layer l."""
    from cascade_token_head_b200.synth import linear_decode_keep
    total = 0.0
    for s in range(w.steps):
        ks = linear_decode_keep(w.T0 + s + 1, w.L)
        for l in range(w.L):
            total += w.B * w.H * ks[l] * w.d_h * 2 + refetch_rows[s][l] * ks[l] * w.d_h + w.B * ks[l] * 4
    return total


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


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------------
# CPU oracle on bounded samples
# ------------------------------------------------------------------------------------------------
def _bf16_values(a):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def oracle_prefill_sample(w, d, seconds: float, max_units: int | None = None):
    """BERT-shaped prefill: the float64 oracle cascade one whole sequence at a time until `seconds`
    elapsed (at least one).  Long-context prefill (one sequence of 16384 tokens is minutes of
    oracle work): the oracle's layer-0 attention of whole heads (all query rows, in row blocks),
    extrapolated to the step by the ratio of the step's attention flops to the sample's.
    Returns (tokens/s, description, threads, seconds spent on the sampled units)."""
    import numpy as np
    from oracle import spatten_ref as R

    wq = [_bf16_values(a) for a in d["w_qkv"]]
    wo = [_bf16_values(a) for a in d["w_o"]]
    done, t0 = 0, time.perf_counter()
    if w.T <= 4096:
        while True:
            b = done % w.B
            X = _bf16_values(d["X"][b:b + 1])
            g = None if d["key_gain"] is None else d["key_gain"][b:b + 1]
            R.cascade_prefill(X, wq, wo, w.H, w.d_h, w.token_keep, w.head_keep, w.quant, w.theta, key_gain=g)
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds or (max_units and done >= max_units):
                break
        return done * w.T / el, f"{done} sequence(s) of the workload (T={w.T}, all {w.L} layers), {el:.1f} s", \
            blas_threads(), el
    X = _bf16_values(d["X"][0])
    qkv = X @ wq[0]
    HD = w.H * w.d_h
    sm = 1.0 / math.sqrt(w.d_h)
    gain = d["key_gain"][0].astype(np.float32)[:, None]
    # units: blocks of 1024 query rows of one head (all keys), heads in turn; a head's K/V are
    # quantized when its first block is taken
    n_blk = (w.T + 1023) // 1024
    cur_h, rows = -1, 0
    t0 = time.perf_counter()
    while True:
        h, r0 = (done // n_blk) % w.H, (done % n_blk) * 1024
        c = slice(h * w.d_h, (h + 1) * w.d_h)
        if h != cur_h:
            kq = R.quantize_head(qkv[:, HD:2 * HD][:, c].astype(np.float32) * gain)
            vq = R.quantize_head(qkv[:, 2 * HD:][:, c].astype(np.float32))
            cur_h = h
        R.progressive_attention(qkv[r0:r0 + 1024, c], kq, vq, w.theta, sm)
        rows += min(1024, w.T - r0)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_units and done >= max_units):
            break
    sample_flops = 4.0 * rows * w.T * w.d_h
    scale = attention_flops(w) / sample_flops
    return w.T / (el * scale), (f"layer-0 attention of {done} block(s) of up to 1024 query rows of one head "
                                f"(all {w.T} keys), {el:.1f} s, extrapolated x{scale:.0f} by attention flops "
                                f"to one step"), blas_threads(), el


def kept_set_report(ctx, S, cfg, W, io, ws, w, d, kept_tok, kept_head, free_running: int = 2, near: float = 1e-5):
    """The comparison protocol for kept sets, on one traced forward of the same inputs (outside the
    timed region):
    - teacher-forced, every sequence and selection: the oracle's top-k over the device's own
      cumulative importance (traced at each selection) must give the device's next kept tokens and
      heads exactly;
    - free-running, `free_running` sequences: the float64 oracle cascade's kept sets against the
      device's, layer by layer up to the first divergence. Each disagreeing token or head is logged
      with its oracle score and the k-th score; it is a near-tie when within `near` (relative) of
      the k-th score. bf16 rounding of the device's activations moves importance by more than
      1e-5, so free-running bf16 disagreements beyond near-ties are reported, not failed."""
    import numpy as np
    from oracle import spatten_ref as R
    torch = ctx.torch
    B, T, H, L = w.B, w.T, w.H, w.L
    ti = torch.zeros((L, B, T), dtype=torch.float32, device=ctx.dev)
    hi = torch.zeros((L, B, H), dtype=torch.float32, device=ctx.dev)
    io.trace_tok_imp, io.trace_head_imp = ti.data_ptr(), hi.data_ptr()
    try:
        S.cascade_forward(cfg, W, io, ws, ws.numel(), stream=ctx.stream)
        torch.cuda.synchronize()
    finally:
        io.trace_tok_imp = io.trace_head_imp = None
    kt, kh = kept_tok.cpu().numpy(), kept_head.cpu().numpy()
    ti, hi = ti.cpu().numpy(), hi.cpu().numpy()
    tf_sel, tf_bad = 0, 0
    for l in range(L - 1):
        k, k2, Hl, H2 = w.token_keep[l], w.token_keep[l + 1], w.head_keep[l], w.head_keep[l + 1]
        for b in range(B):
            kl = kt[l, b, :k]
            want = kl[R.topk_select(ti[l, b, kl].astype(np.float64), k2)]
            tf_bad += int(not np.array_equal(want, kt[l + 1, b, :k2]))
            hl = kh[l, b, :Hl]
            want_h = hl[R.topk_select(hi[l, b, hl].astype(np.float64), H2)]
            tf_bad += int(not np.array_equal(want_h, kh[l + 1, b, :H2]))
            tf_sel += 2
    wq = [_bf16_values(a) for a in d["w_qkv"]]
    wo = [_bf16_values(a) for a in d["w_o"]]
    log, near_ties, other, first_div = [], 0, 0, []
    for b in range(min(free_running, B)):
        g = None if d["key_gain"] is None else d["key_gain"][b:b + 1]
        r = R.cascade_prefill(_bf16_values(d["X"][b:b + 1]), wq, wo, H, w.d_h, w.token_keep, w.head_keep, w.quant,
                              w.theta, key_gain=g)
        div = None
        for l in range(1, L):
            for kind, dev_set, ora_set, scores, kk in (
                    ("token", kt[l, b, :w.token_keep[l]], r["kept"][l][0], r["I_sel"][l - 1][0], w.token_keep[l]),
                    ("head", kh[l, b, :w.head_keep[l]], r["heads"][l][0], r["J_sel"][l - 1][0], w.head_keep[l])):
                a_only = np.setdiff1d(ora_set, dev_set)
                d_only = np.setdiff1d(dev_set, ora_set)
                if a_only.size == 0 and d_only.size == 0:
                    continue
                prev = r["kept"][l - 1][0] if kind == "token" else r["heads"][l - 1][0]
                ranked = np.sort(scores[prev])[::-1]
                kth = float(ranked[kk - 1])
                for t in np.concatenate([a_only, d_only]):
                    tie = abs(float(scores[t]) - kth) <= near * abs(kth)
                    near_ties += int(tie)
                    other += int(not tie)
                    if len(log) < 20:
                        log.append({"sequence": b, "layer": l, "kind": kind, "id": int(t),
                                    "in": "oracle" if t in a_only else "device", "oracle_score": float(scores[t]),
                                    "kth_score": kth, "near_tie": bool(tie)})
                div = l
            if div is not None:
                break
        first_div.append(div)
    return {"teacher_forced": {"sequences": B, "selections": tf_sel, "mismatches": tf_bad},
            "free_running": {"sequences": min(free_running, B), "first_divergence_layer": first_div,
                             "near_tie_disagreements": near_ties, "other_disagreements": other, "log": log,
                             "note": "float64 oracle on the bf16 inputs and weights; the device keeps bf16 "
                                     "activations, so disagreements beyond near-ties are expected and reported"}}


class OracleDecode:
    """The float64 oracle generating tokens of the decode workload, for the CPU baseline."""

    def __init__(self, w, d):
        from oracle import spatten_ref as R
        self.R, self.w = R, w
        self.wq = [_bf16_values(a) for a in d["w_qkv"]]
        self.wo = [_bf16_values(a) for a in d["w_o"]]
        self.caches = R.empty_decode_caches(len(self.wq), w.B, w.H, w.cap, w.d_h)
        for l, c in enumerate(self.caches):
            R.quantize_prompt_cache(c, d["k_prompt"][l], d["v_prompt"][l])
        self.xs = d["x_steps"]

    def generate(self, seconds: float, max_tokens: int | None = None):
        """Generate tokens (teacher-forced inputs x_t, all sequences) from the prompt until
        `seconds` elapsed.  Returns (generated tokens/s, tokens per sequence, wall seconds)."""
        import numpy as np
        from cascade_token_head_b200.synth import linear_decode_keep
        w, R = self.w, self.R
        n_old, I = w.T0, np.zeros((w.B, w.cap))
        done, t0 = 0, time.perf_counter()
        L = len(self.wq)
        while True:
            R.decode_step(_bf16_values(self.xs[done % w.steps]), self.caches, n_old, I, self.wq, self.wo,
                          w.H, w.d_h, lambda n: linear_decode_keep(n, L), w.theta)
            n_old += 1
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds or (max_tokens and done >= max_tokens) or n_old >= w.cap:
                break
        return done * w.B / el, done, el


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from cascade_token_head_b200 import synth
    steps = max(1, args.steps)
    # every step is one bounded unit of the workload: warm-up and timed runs take exactly
    # args.warmup and `steps` units (no time budget)
    if args.workload == "gpt2m_decode":
        w = synth.gpt2m_decode()
        o = OracleDecode(w, synth.draw_decode(w))
        if args.warmup > 0:
            o.generate(math.inf, max_tokens=args.warmup)
        t0 = time.perf_counter()
        _, done, _ = o.generate(math.inf, max_tokens=steps)
        el = time.perf_counter() - t0
        value = done * w.B / el
        cfg = {"workload": w.name, "global_batch": w.B, "prompt_len": w.T0, "parallelism": "replicas"}
        sample = f"one generated token of all {w.B} sequences (all {w.L} layers) per step, {done} steps"
    else:
        w = prefill_workload(args.workload)
        d = synth.draw_prefill(w)
        if args.warmup > 0:
            oracle_prefill_sample(w, d, math.inf, max_units=args.warmup)
        value, sample, _, el = oracle_prefill_sample(w, d, math.inf, max_units=steps)
        cfg = {"workload": w.name, "global_batch": w.B, "seq_len": w.T, "parallelism": "replicas"}
        unit = "one sequence" if w.T <= 4096 else "one 1024-row block of one head's layer-0 attention"
        sample = f"{unit} per step ({sample})"
    line = {"metric": METRIC[args.workload], "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
class Ranks:
    """Rank identity (RANK / WORLD_SIZE / LOCAL_RANK from the launcher) and the only collectives the
    bench takes: a barrier and a max over ranks of a device time.  No collective touches the data
    path; each rank runs its own sequences (seeded by its rank).  backend "nccl" with a CUDA device
    on the GPU, "gloo" with the CPU (tests)."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: int = 120):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device if device is not None else torch.device("cpu")
        if self.world > 1:
            from datetime import timedelta
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, v: float) -> float:
        if self.world == 1:
            return v
        t = self.torch.tensor([v], dtype=self.torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, max_total_ms: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank_step per step, and the
    job takes the slowest rank's time (weak scaling)."""
    return world * units_per_rank_step * steps / (max_total_ms / 1e3)


class Ctx(Ranks):
    """Device, ranks, stream and the L2 flush buffer shared by the workloads."""

    def __init__(self):
        import torch
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        super().__init__("nccl", torch.device("cuda", local))
        self.dev = self.device
        self.stream = torch.cuda.current_stream()
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=self.dev)

    def events(self, n):
        """n timing events, materialised on the stream so their handles can be handed over."""
        ev = [self.torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in ev:
            e.record(self.stream)
        return ev


def timed_replays(ctx, replay, K, after_each):
    """K timed replays bracketed by events, an L2 flush before each (outside the events), clocks
    sampled throughout.  after_each(i) runs after the replay has finished (reads its events)."""
    torch = ctx.torch
    ev_s, ev_e = ctx.events(K), ctx.events(K)
    clocks = ClockSampler(ctx.local)
    ctx.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for i in range(K):
        ctx.flush.zero_()
        ev_s[i].record(ctx.stream)
        replay()
        ev_e[i].record(ctx.stream)
        torch.cuda.synchronize()
        after_each(i)
    clk = clocks.stop()
    ctx.barrier()
    total_ms = ctx.max_over_ranks(sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(K)))
    return total_ms, clk


def e2e_loop(ctx, body, n):
    """Device-timed iterations of `body` (host->device copy, forward, device->host copy)."""
    torch = ctx.torch
    ms = []
    for _ in range(n):
        ctx.flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(ctx.stream)
        body()
        b.record(ctx.stream)
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    return ctx.max_over_ranks(sum(ms)), n


def e2e_pipelined(ctx, slots, x_host, gain_host, forward, n):
    """n consecutive steps, device-timed together (L2 flushed once before): step i's inputs are copied
    into slot i % 2 on a copy stream while step i - 1 runs, and its outputs are copied out on the
    same stream while step i + 1 runs.  Returns the total milliseconds (max over ranks)."""
    torch = ctx.torch
    copy = torch.cuda.Stream(device=ctx.dev)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    fwd_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def copy_in(j, after_fwd):
        xj, gj = slots[j][0], slots[j][1]
        with torch.cuda.stream(copy):
            if after_fwd is not None:
                copy.wait_event(after_fwd)   # the slot's inputs were read by that step's forward
            xj.copy_(x_host, non_blocking=True)
            gj.copy_(gain_host, non_blocking=True)
            h2d_done[j].record(copy)

    ctx.flush.zero_()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(ctx.stream)
    copy.wait_stream(ctx.stream)
    copy_in(0, None)
    for i in range(n):
        j = i % 2
        if i + 1 < n:
            copy_in((i + 1) % 2, fwd_done[(i + 1) % 2] if i >= 1 else None)
        ctx.stream.wait_event(h2d_done[j])
        if i >= 2:
            ctx.stream.wait_event(d2h_done[j])   # the slot's outputs of step i - 2 have been copied out
        forward(slots[j][3])
        fwd_done[j].record(ctx.stream)
        with torch.cuda.stream(copy):
            copy.wait_event(fwd_done[j])
            for dev_t, host_t in zip(slots[j][2], slots[j][4]):
                host_t.copy_(dev_t, non_blocking=True)
            d2h_done[j].record(copy)
    ctx.stream.wait_stream(copy)
    b.record(ctx.stream)
    torch.cuda.synchronize()
    return ctx.max_over_ranks(a.elapsed_time(b))


def prefill_arm(ctx, args, name):
    import numpy as np
    torch = ctx.torch
    from cascade_token_head_b200 import spatten as S
    from cascade_token_head_b200 import synth

    w = prefill_workload(name)
    w.seed = ctx.rank
    d = synth.draw_prefill(w)
    bf, dev = torch.bfloat16, ctx.dev
    B, T, D, H, L = w.B, w.T, w.D, w.H, w.L
    X_host = torch.from_numpy(d["X"]).to(bf).pin_memory()
    gain_host = torch.from_numpy(d["key_gain"].astype(np.float32)).pin_memory()
    X = X_host.to(dev)
    gain = gain_host.to(dev)
    W = [(torch.from_numpy(d["w_qkv"][l]).to(bf).to(dev), torch.from_numpy(d["w_o"][l]).to(bf).to(dev))
         for l in range(L)]
    x_out = torch.empty((B, w.token_keep[-1], D), dtype=bf, device=dev)
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

    def step():
        S.cascade_forward(cfg, W, io, ws, ws.numel(), stream=ctx.stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status after warm-up"

    # the library records event pair (2l, 2l+1) around layer l's attention launches; inside the
    # captured step they become event-record nodes of the graph
    attn_ev = ctx.events(2 * L)
    torch.cuda.synchronize()
    attn_array = (C.c_void_p * (2 * L))(*[e.cuda_event for e in attn_ev])
    io.attn_events = C.cast(attn_array, C.POINTER(C.c_void_p))
    graph, launches_per_step = None, None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        l0 = S.kernel_launch_count()
        with torch.cuda.graph(graph):
            S.cascade_forward(cfg, W, io, ws, ws.numel(), stream=torch.cuda.current_stream())
        launches_per_step = S.kernel_launch_count() - l0
        graph.replay()
        torch.cuda.synchronize()
    K = args.steps
    attn_ms = []
    launches0 = S.kernel_launch_count()
    total_ms, clk = timed_replays(
        ctx, graph.replay if graph is not None else step, K,
        lambda i: attn_ms.append(sum(attn_ev[2 * l].elapsed_time(attn_ev[2 * l + 1]) for l in range(L))))
    launches = launches_per_step * K if graph is not None else S.kernel_launch_count() - launches0
    io.attn_events = None
    assert int(status.item()) == 0, "device status after timing"
    refetch_rows = refetch.cpu().tolist()

    # end to end through the C ABI with host buffers: every step copies X and key_gain in from pinned
    # host memory, runs spatten_cascade_forward (direct launches) and copies the final rows, the
    # kept sets and the cumulative importance out; the copies of neighbouring steps overlap the
    # forward on a second stream (two sets of device inputs and outputs)
    h2d = X_host.numel() * X_host.element_size() + gain_host.numel() * 4
    d2h = x_out.numel() * 2 + kept_tok.numel() * 4 + tok_imp.numel() * 4
    slots = []
    for j in range(2):
        xj = X if j == 0 else torch.empty_like(X)
        gj = gain if j == 0 else torch.empty_like(gain)
        oj = (x_out, kept_tok, tok_imp) if j == 0 else tuple(torch.empty_like(t) for t in (x_out, kept_tok, tok_imp))
        ioj = S.cascade_io()
        ioj.x, ioj.key_gain, ioj.x_out = xj.data_ptr(), gj.data_ptr(), oj[0].data_ptr()
        ioj.kept_tok, ioj.kept_head = oj[1].data_ptr(), kept_head.data_ptr()
        ioj.tok_imp, ioj.head_imp, ioj.refetch_count = oj[2].data_ptr(), head_imp.data_ptr(), refetch.data_ptr()
        ioj.dev_status = status.data_ptr()
        hosts = tuple(torch.empty_like(t, device="cpu").pin_memory() for t in oj)
        slots.append((xj, gj, oj, ioj, hosts))
    n_e2e = max(3, K)
    e2e_total = e2e_pipelined(ctx, slots, X_host, gain_host,
                              lambda io_j: S.cascade_forward(cfg, W, io_j, ws, ws.numel(), stream=ctx.stream), n_e2e)
    assert int(status.item()) == 0, "device status after the end-to-end loop"
    # the same loop with each slot's forward replayed from a CUDA graph captured from the same call
    e2e_graph_total = None
    if graph is not None:
        slot_graphs = []
        for slot in slots:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                S.cascade_forward(cfg, W, slot[3], ws, ws.numel(), stream=torch.cuda.current_stream())
            slot_graphs.append(g)
        torch.cuda.synchronize()
        e2e_graph_total = e2e_pipelined(ctx, slots, X_host, gain_host,
                                        lambda io_j: slot_graphs[0 if io_j is slots[0][3] else 1].replay(), n_e2e)
        assert int(status.item()) == 0, "device status after the graph end-to-end loop"
    tokens_per_step = B * T
    peaks, peak_kind = load_peaks()
    flops = attention_flops(w)
    attn_s = statistics.mean(attn_ms) / 1e3
    achieved = flops / attn_s / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    traffic, traffic_src = prefill_traffic(w)
    result = {
        "metric": METRIC[name],
        "value": whole_job_rate(ctx.world, tokens_per_step, K, total_ms), "unit": "tokens/s", "n_gpus": ctx.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": w.name, "global_batch": B * ctx.world, "seq_len": T, "d_model": D, "heads": H,
                   "layers": L, "token_keep": w.token_keep, "head_keep": w.head_keep, "refetch_threshold": w.theta,
                   "parallelism": f"dp{ctx.world} (independent sequences)", "l2": "flushed between timed steps",
                   "launch": "CUDA graph of one step" if graph is not None else "direct launches"},
        "roofline": {"kernel": "attention (spatten_attention_layer kernels, all layers)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16 sustained (the MMAs take fp16 operands: same nominal "
                                  f"dense rate, ratio 1)", "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_flops_per_step": flops, "attn_ms_per_step": attn_s * 1e3},
        "e2e": {"value": whole_job_rate(ctx.world, tokens_per_step, n_e2e, e2e_total), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "method": f"{n_e2e} consecutive steps timed together, each a direct spatten_cascade_forward "
                          f"call; each step's copies in and out on a second stream, overlapping the "
                          f"neighbouring steps' forward",
                "graph_value": (whole_job_rate(ctx.world, tokens_per_step, n_e2e, e2e_graph_total)
                                if e2e_graph_total else None),
                "graph_method": "the same loop, each step's forward replayed from a CUDA graph captured from "
                                "the same call"},
        "gpu_launches": int(launches),
        "clocks": clk,
        "refetch_rows_per_layer": refetch_rows,
    }
    if ctx.rank == 0 and not args.no_kept_report and w.T <= 4096:
        result["kept_sets"] = kept_set_report(ctx, S, cfg, W, io, ws, w, d, kept_tok, kept_head)
    if ctx.rank == 0 and not args.no_cpu_baseline:
        v, sample, threads, _ = oracle_prefill_sample(w, d, args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                  "sample": sample}
    return result


def decode_arm(ctx, args, steps):
    torch = ctx.torch
    from cascade_token_head_b200 import spatten as S
    from cascade_token_head_b200 import synth
    from cascade_token_head_b200.decode import DecodeState

    w = synth.gpt2m_decode()
    w.seed = ctx.rank
    d = synth.draw_decode(w)
    st = DecodeState(w, d["w_qkv"], d["w_o"], d["k_prompt"], d["v_prompt"])
    torch.cuda.synchronize()
    bf, dev, L = torch.bfloat16, ctx.dev, w.L
    xs_host = torch.from_numpy(d["x_steps"]).to(bf).pin_memory()          # [steps, B, D]
    xs = xs_host.to(dev)
    outs = torch.empty_like(xs)
    outs_host = torch.empty_like(xs_host).pin_memory()
    imp_host = torch.empty_like(st.tok_imp, device="cpu").pin_memory()
    refetch = torch.zeros((w.steps, L), dtype=torch.int32, device=dev)
    attn_ev = [ctx.events(2 * L) for _ in range(w.steps)]
    torch.cuda.synchronize()
    arrays = [(C.c_void_p * (2 * L))(*[e.cuda_event for e in row]) for row in attn_ev]

    def generation(timed_events):
        st.reset()
        for s in range(w.steps):
            st.step(x=xs[s], x_out=outs[s], refetch=refetch[s], events=arrays[s] if timed_events else None,
                    stream=torch.cuda.current_stream())

    for _ in range(args.warmup):
        generation(False)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0, "device status after warm-up (decode)"
    graph = torch.cuda.CUDAGraph()
    l0 = S.kernel_launch_count()
    with torch.cuda.graph(graph):
        generation(True)
    launches_per_gen = S.kernel_launch_count() - l0
    graph.replay()
    torch.cuda.synchronize()
    attn_ms = []
    total_ms, clk = timed_replays(
        ctx, graph.replay, steps,
        lambda i: attn_ms.append(sum(row[2 * l].elapsed_time(row[2 * l + 1]) for row in attn_ev for l in range(L))))
    assert int(st.status.item()) == 0, "device status after timing (decode)"
    refetch_rows = refetch.cpu().tolist()

    def e2e_body():
        xs.copy_(xs_host, non_blocking=True)
        generation(False)
        outs_host.copy_(outs, non_blocking=True)
        imp_host.copy_(st.tok_imp, non_blocking=True)

    e2e_total, n_e2e = e2e_loop(ctx, e2e_body, 2)
    tokens = w.B * w.steps
    peaks, peak_kind = load_peaks()
    nbytes = decode_attention_bytes(w, refetch_rows)
    attn_s = statistics.mean(attn_ms) / 1e3
    achieved = nbytes / attn_s / 1e9
    peak = float(peaks.get("hbm_gbs"))
    all_rows = w.B * w.H * w.steps * L
    result = {
        "metric": METRIC["gpt2m_decode"],
        "value": whole_job_rate(ctx.world, tokens, steps, total_ms), "unit": "tokens/s", "n_gpus": ctx.world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": total_ms / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": w.name, "global_batch": w.B * ctx.world, "prompt_len": w.T0,
                   "generated_per_step": w.steps, "d_model": w.D, "heads": w.H, "layers": L,
                   "keep": "linear to 50 % of the cache rows by the last layer", "refetch_threshold": w.theta,
                   "parallelism": f"dp{ctx.world} (independent sequences)", "l2": "flushed between timed steps",
                   "launch": "CUDA graph of one 128-token generation"},
        "roofline": {"kernel": "decode attention (spatten_attention_layer decode kernel, all layers and tokens)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} HBM copy", "traffic": None,
                     "algorithmic_bytes_per_step": nbytes, "attn_ms_per_step": attn_s * 1e3},
        "e2e": {"value": whole_job_rate(ctx.world, tokens, n_e2e, e2e_total), "unit": "tokens/s",
                "h2d_bytes_per_step": xs_host.numel() * 2,
                "d2h_bytes_per_step": outs_host.numel() * 2 + imp_host.numel() * 4},
        "gpu_launches": int(launches_per_gen * steps),
        "clocks": clk,
        "refetched_row_fraction": sum(map(sum, refetch_rows)) / all_rows,
    }
    if ctx.rank == 0 and not args.no_cpu_baseline:
        o = OracleDecode(w, d)
        v, n, el = o.generate(args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                  "sample": f"{n} generated token(s) of all {w.B} sequences (all {L} layers), "
                                            f"{el:.1f} s"}
    return result


def graph_of(ctx, call):
    """A CUDA graph of one call (captured after one direct run), and the library kernels it launches."""
    from cascade_token_head_b200 import spatten as S
    torch = ctx.torch
    call(ctx.stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    l0 = S.kernel_launch_count()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    launches = S.kernel_launch_count() - l0
    g.replay()
    torch.cuda.synchronize()
    return g, launches


def hbm_entry(ctx, args, call, nbytes, h2d, d2h, what):
    """Device time of one call (graph replays, L2 flushed between), its HBM roofline over the
    algorithmic bytes, and the same call end to end with its host copies (e2e_body)."""
    torch = ctx.torch
    g, launches = graph_of(ctx, call)
    K = max(5, args.steps)
    for _ in range(3):
        g.replay()
    total_ms, clk = timed_replays(ctx, g.replay, K, lambda i: None)
    t = total_ms / K / 1e3
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("hbm_gbs"))
    achieved = nbytes / t / 1e9
    e2e_ms, n = e2e_loop(ctx, lambda: (h2d(), g.replay(), d2h()), 3)
    return {"us_per_call": t * 1e6, "gpu_launches_per_call": int(launches),
            "roofline": {"kernel": what, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": f"{peak_kind} HBM copy", "traffic": None,
                         "algorithmic_bytes_per_call": nbytes},
            "e2e_ms_per_call": e2e_ms / n, "clocks": clk}


def topk_arm(ctx, args):
    """The top-k sweep's long rows: 64 rows of N in {256k, 1M} keys, k = 10 % and 50 %, uniform and
    lognormal values with 1 % exact duplicates.  GB/s over the algorithmic bytes 64 (4N + 4k)."""
    import numpy as np
    torch = ctx.torch
    from cascade_token_head_b200 import spatten as S
    from cascade_token_head_b200 import synth
    R_, entries = 64, []
    for N in (262144, 1048576):
        for dist in ("uniform", "lognormal"):
            x_np = synth.draw_topk_row_block(R_, N, dist, 0.01, seed=N % 9973 + (dist == "lognormal") + 100 * ctx.rank)
            x_host = torch.from_numpy(x_np).pin_memory()
            x = x_host.to(ctx.dev)
            for frac in (0.1, 0.5):
                k = int(frac * N)
                out = torch.empty((R_, k), dtype=torch.int32, device=ctx.dev)
                out_host = torch.empty((R_, k), dtype=torch.int32).pin_memory()
                nb = S.topk_workspace_size(R_, N, k)
                wsb = torch.empty(max(nb, 16), dtype=torch.uint8, device=ctx.dev)
                call = lambda st, x=x, out=out, k=k, wsb=wsb, nb=nb: S.topk_select(
                    x, R_, N, N, k, out, k, ws=wsb, ws_bytes=nb, stream=st)
                e = hbm_entry(ctx, args, call, R_ * (4.0 * N + 4.0 * k),
                              lambda x=x, x_host=x_host: x.copy_(x_host, non_blocking=True),
                              lambda out=out, out_host=out_host: out_host.copy_(out, non_blocking=True),
                              "spatten_topk_select (all of its launches)")
                n_b = N * R_ * 4
                e.update(N=N, k=k, dist=dist, value=R_ * (4.0 * N + 4.0 * k) / (e["us_per_call"] / 1e6) / 1e9,
                         unit="GB/s",
                         e2e={"value": R_ * (4.0 * N + 4.0 * k) / (e.pop("e2e_ms_per_call") / 1e3) / 1e9,
                              "unit": "GB/s", "h2d_bytes_per_step": n_b, "d2h_bytes_per_step": R_ * k * 4})
                if ctx.rank == 0 and not args.no_cpu_baseline:
                    from oracle import spatten_ref as R
                    t0, rows = time.perf_counter(), 0
                    while rows < R_ and (rows == 0 or time.perf_counter() - t0 < 1.0):
                        R.topk_select(x_np[rows].astype(np.float64), k)
                        rows += 1
                    el = time.perf_counter() - t0
                    e["cpu_baseline"] = {"value": rows * (4.0 * N + 4.0 * k) / el / 1e9, "unit": "GB/s", "cores": 1,
                                         "kind": "oracle", "sample": f"{rows} row(s) of the 64, {el:.2f} s"}
                entries.append(e)
                del out, wsb
            del x
    head = next(e for e in entries if e["N"] == 1048576 and e["k"] == 524288 and e["dist"] == "uniform")
    return {"metric": "top-k select GB/s (64 rows, ascending indices, ties to the lower index)", "unit": "GB/s",
            "value": head["value"], "config": {"workload": "topk_sweep_long_rows", "rows": R_,
                                               "l2": "flushed between timed calls"},
            "roofline": head["roofline"], "entries": entries}


def gather_arm(ctx, args):
    """Kept-row gathers of the two prefill workloads' X (bf16 rows): BERT-base layer 0 -> 1
    (32 x 461 of 512 rows of 1536 B) and long-context layer 0 -> 1 (8192 of 16384 rows of 8192 B).
    GB/s over the algorithmic bytes k (2 row_bytes + 4)."""
    import numpy as np
    torch = ctx.torch
    from cascade_token_head_b200 import spatten as S
    from cascade_token_head_b200 import synth
    entries = []
    for name, B, n, D, k in (("bert_base_x_rows", 32, 512, 768, 461), ("long_context_x_rows", 1, 16384, 4096, 8192)):
        g = synth.rng_for(7 + ctx.rank)
        src_host = torch.from_numpy(g.standard_normal((B, n, D)).astype(np.float32)).to(torch.bfloat16).pin_memory()
        idx_np = np.stack([np.sort(g.choice(n, k, replace=False)) for _ in range(B)]).astype(np.int32)
        src = src_host.to(ctx.dev)
        idx = torch.from_numpy(idx_np).to(ctx.dev)
        dst = torch.empty((B, k, D), dtype=torch.bfloat16, device=ctx.dev)
        dst_host = torch.empty((B, k, D), dtype=torch.bfloat16).pin_memory()
        rb = D * 2
        call = lambda st, src=src, idx=idx, dst=dst, B=B, n=n, k=k, rb=rb: S.gather_kept(
            src, n * rb, rb, n, rb, B, idx, k, k, dst, k * rb, rb, stream=st)
        nbytes = B * k * (2.0 * rb + 4)
        e = hbm_entry(ctx, args, call, nbytes, lambda src=src, src_host=src_host: src.copy_(src_host, non_blocking=True),
                      lambda dst=dst, dst_host=dst_host: dst_host.copy_(dst, non_blocking=True),
                      "spatten_gather_kept")
        torch.cuda.synchronize()
        assert np.array_equal(dst[0].view(torch.int16).cpu().numpy(),
                              src_host[0].view(torch.int16).numpy()[idx_np[0]]), "gathered rows"
        e.update(name=name, rows=B * k, row_bytes=rb, value=nbytes / (e["us_per_call"] / 1e6) / 1e9, unit="GB/s",
                 e2e={"value": nbytes / (e.pop("e2e_ms_per_call") / 1e3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": B * n * rb, "d2h_bytes_per_step": B * k * rb})
        if ctx.rank == 0 and not args.no_cpu_baseline:
            xs = src_host.view(torch.int16).numpy()
            t0, reps = time.perf_counter(), 0
            while reps == 0 or time.perf_counter() - t0 < 0.5:
                for b in range(B):
                    np.take(xs[b], idx_np[b], axis=0)
                reps += 1
            el = time.perf_counter() - t0
            e["cpu_baseline"] = {"value": reps * nbytes / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "numpy take",
                                 "sample": f"{reps} full gather(s), {el:.2f} s"}
        entries.append(e)
        del src, dst
    head = entries[0]
    return {"metric": "kept-row gather GB/s", "unit": "GB/s", "value": head["value"],
            "config": {"workload": "prefill_x_row_gathers", "l2": "flushed between timed calls"},
            "roofline": head["roofline"], "entries": entries}


def sub_line(r, keys=("metric", "value", "unit", "steps", "ms_per_step", "config", "roofline", "e2e", "gpu_launches",
                      "clocks", "refetched_row_fraction", "refetch_rows_per_layer", "cpu_baseline")):
    return {k: r[k] for k in keys if k in r}


def run_ours(args):
    ctx = Ctx()
    if args.workload == "gpt2m_decode":
        result = decode_arm(ctx, args, args.steps)
    else:
        result = prefill_arm(ctx, args, args.workload)
        if args.workload == "bert_base_prefill" and not args.no_extra:
            result["decode"] = sub_line(decode_arm(ctx, args, max(3, args.steps // 4)))
            long_args = argparse.Namespace(**{**vars(args), "steps": max(3, args.steps // 4),
                                              "cpu_seconds": min(args.cpu_seconds, 8.0)})
            result["long_prefill"] = sub_line(prefill_arm(ctx, long_args, "long_prefill"))
            result["topk_sweep"] = topk_arm(ctx, args)
            result["gather"] = gather_arm(ctx, args)
    ctx.close()
    if ctx.rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def relaunch_with_ranks(args, argv):
    """`--gpus N` without a launcher: run N local ranks (one per GPU) under torch.distributed.run on
    127.0.0.1, the way the multi-GPU runs are launched; rank 0 prints the line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(METRIC), default="bert_base_prefill")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", "--no-decode", action="store_true",
                    help="leave the decode, long_prefill, topk_sweep and gather objects out of the default line")
    ap.add_argument("--no-kept-report", action="store_true",
                    help="skip the kept-set comparison against the oracle (teacher-forced and free-running)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the prefill step directly instead of replaying a CUDA graph")
    args = ap.parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_with_ranks(args, sys.argv[1:] if argv is None else list(argv))
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) != args.gpus:
        print(f"warning: --gpus {args.gpus} but the launcher started {os.environ['WORLD_SIZE']} ranks", file=sys.stderr)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    raise SystemExit(main())
