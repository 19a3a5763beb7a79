"""Benchmark of the TokenGate gated-prefill hot path on B200.

One step = gate score (all N tokens) -> top-K select -> gather/compaction ->
one token-gated decoder layer on the M kept rows, on the Qwen3-1.7B-shaped
single-layer workload (N = 16384 tokens of which the last 64 are the question,
d_model 2048, GQA 16/8 x 128, gate MLP 2048 -> 256 -> 1, K = 2000, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  Multi-GPU runs are independent replicas (one
request per GPU, no collective on the data path): value = all tokens / the
slowest rank's time.  `--impl reference` times the CPU oracle on the host
cores instead (bounded sample per step).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import types
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-prefill tokens/s & TTFT ms at N=16K/128K; attention % bf16 peak"
L2_FLUSH_BYTES = 256 << 20   # > the 126 MB L2

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, from
# an ncu capture of `bench.py --ncu-case` (its summary is kept under profiles/),
# with the rows that launch processed; scaled to the bench launch by rows.  A
# record counts only while the SHA-256 of its kernel's sources still matches.
MEASURED_TRAFFIC = {
    "linear_gate_up_swiglu": {"bytes": 58823680 + 8841472, "rows": 2064, "sources": ("gemm_tc.cuh", "common.cuh"),
                              "sha256": "527a8b39fc28c7c0d19969704ccff730efd0618e8420255ad1f826e8c2b07b6b"},
    "gate_score": {"bytes": 269996544 + 6056704, "rows": 65536, "sources": ("gate_tc.cuh", "common.cuh"),
                   "sha256": "119cea418d54f0b167a567331415219d357f7a3e836c5eeb503578c143718edb"},
    "attention": {"bytes": 17002240 + 0, "rows": 2064, "sources": ("attn_tc.cuh", "common.cuh"),
                  "sha256": "dea1b84a1dcf77b3a2579da49c6d3c8937eb553f075a054d4d52c78a1f465801"},
}


# ----------------------------------------------------------------------------- helpers (host only)

def measured_traffic(kernel: str, rows: int):
    """Per-launch DRAM traffic of `kernel` at `rows` rows, or None when no
    capture exists or its sources changed since the capture."""
    import hashlib
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        with open(os.path.join(ROOT, "learned_token_pruning_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != rec["sha256"]:
        return None
    return rec["bytes"] * rows / rec["rows"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def workload_work(w, m):
    """Algorithmic bytes / flops of each call of one step: the gate reads every
    hidden row once (plus mask, score and W1), the selector its scores and mask
    and writes the kept indices, the gather reads and writes each kept row
    (the fused gather + RMSNorm writes it twice), attention counts the kept
    causal pairs times the two contractions, each GEMM 2*M*K*N."""
    n, dm, h, D, hq, hkv, dff = w.n, w.d_model, w.gate_hidden, w.head_dim, w.hq, w.hkv, w.d_ff
    es = 2 if w.dtype == "bf16" else 4
    qkv = (hq + 2 * hkv) * D
    return {
        "gate_score": {"bytes": n * dm * es + n * 1 + n * 4 + h * dm * es, "flops": 2 * n * dm * h},
        "topk_select": {"bytes": n * 4 + n * 1 + m * 4},
        # the fused call: the gate's bytes plus the selector's (scores and mask read back, indices written)
        "gate_score_select": {"bytes": n * dm * es + n * 1 + n * 4 + h * dm * es + n * 4 + n * 1 + m * 4},
        "unfused_gather": {"bytes": 2 * m * dm * es + m * 4 * 5},
        "gather_rmsnorm": {"bytes": 3 * m * dm * es + m * 4 * 5 + dm * 4},
        "attention": {"flops": 2 * D * hq * m * (m + 1)},
        "linear_qkv": {"flops": 2 * m * dm * qkv},
        "linear_o": {"flops": 2 * m * hq * D * dm},
        "linear_gate_up_swiglu": {"flops": 2 * m * dm * 2 * dff},
        "linear_down": {"flops": 2 * m * dff * dm},
    }


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    couple of milliseconds from a host thread while the timed region runs (the
    step is short, so nvidia-smi's 200 ms polling would see none of it)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_uuid: str, fallback_index: int, period_s: float = 0.002):
        import threading
        self.samples, self.reasons, self.max_mhz, self.error = [], set(), None, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            try:
                self.h = nv.nvmlDeviceGetHandleByUUID(device_uuid)
            except nv.NVMLError:
                self.h = nv.nvmlDeviceGetHandleByIndex(fallback_index)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:             # no NVML: the line says so instead of a clock record
            self.error = f"{type(e).__name__}: {e}"
            return
        self.period = period_s
        self._thread = threading.Thread(target=self._run, daemon=True)

    def start(self):
        if self._thread is not None:
            self._thread.start()

    def sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for name, const in self.REASONS:
            if bits & getattr(nv, const, 0):
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.sample()
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            self._stop.wait(self.period)

    def stop(self):
        if self._thread is None:
            return {"error": self.error} if self.error else None
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return {"error": self.error or "no sample"}
        return {"sm_mhz": statistics.median(self.samples), "sm_min_mhz": min(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml"}


def dist_setup():
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, None
    rank = int(os.environ["RANK"])
    import datetime
    import torch
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, ws, dist


def max_over_ranks(x: float, dist, device=None) -> float:
    """Largest value of x over all ranks (host float in, host float out)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, units_per_step: int, steps: int, slowest_seconds: float) -> float:
    """Whole-job throughput of `world` independent replicas: every rank processes
    units_per_step per step, and the job takes as long as its slowest rank."""
    return world * units_per_step * steps / slowest_seconds


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle timing

def oracle_step_seconds(w, gate_rows: int = 2048):
    """Time the oracle on a bounded sample of one step and scale it to the whole step.

    Sample: gate scores of `gate_rows` tokens (scaled by N / gate_rows), the
    selector on all N scores, the gather and the decoder layer on all M kept
    rows.  Returns (seconds per full step, description, threads).
    """
    from oracle import tokengate_oracle as O
    from learned_token_pruning_b200 import synth
    gate = synth.gate_inputs(w)
    layer = synth.layer_weights(w)
    hp = synth.head_params(w)
    t0 = time.perf_counter()
    s_part = O.gate_scores(gate["hidden"][:gate_rows], gate["norm_w"], 1e-6, gate["w1"], gate["b1"], gate["w2"],
                           gate["b2"], gate["prunable"][:gate_rows])
    t_gate = (time.perf_counter() - t0) * (w.n / gate_rows)
    # full score array for the selector: sampled rows plus the rest drawn from their distribution
    rng = np.random.default_rng(0)
    s = rng.normal(float(np.mean(s_part)), float(np.std(s_part) + 1e-12), size=w.n)
    s[:gate_rows] = s_part
    s[gate["prunable"] == 0] = 0.0
    s32 = s.astype(np.float32)
    t0 = time.perf_counter()
    idx = O.select_kept(s32, gate["prunable"], w.k)
    g = O.gather(gate["hidden"], idx, s32, gate["prunable"], 1e-6)
    t_sel = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.decoder_layer(g["hidden_kept"], layer, hq=w.hq, hkv=w.hkv, head_dim=w.head_dim, pos=g["pos"], bias=g["bias"],
                    ratio=g["ratio"], head_gain=hp["head_gain"], head_temp=hp["head_temp"],
                    rope_theta=w.rope_theta, qk_norm=w.qk_norm)
    t_layer = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    desc = (f"oracle (numpy fp64): gate MLP on {gate_rows} of {w.n} tokens scaled x{w.n / gate_rows:g}, "
            f"selector + gather on all {w.n}, decoder layer on all {idx.size} kept rows")
    return t_gate + t_sel + t_layer, desc, threads


def run_reference(args, w):
    rank, world, dist = dist_setup()
    if dist is not None:
        dist.destroy_process_group()  # rank 0 alone times the oracle; no collective follows
    if rank != 0:
        return
    times = []
    desc, threads = "", 1
    for i in range(args.warmup + args.steps):
        sec, desc, threads = oracle_step_seconds(w)
        if i >= args.warmup:
            times.append(sec)
    step_s = sum(times) / len(times)
    value = w.n / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, world):
    return {"workload": w.name, "n_tokens": w.n, "question_tokens": w.n_question, "k_budget": w.k,
            "kept_rows": w.m, "d_model": w.d_model, "heads": f"{w.hq}/{w.hkv}x{w.head_dim}",
            "gate_mlp": f"{w.d_model}->{w.gate_hidden}->1", "d_ff": w.d_ff, "layers_above_gate": 1,
            "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before every timed step",
            "launch": "one CUDA graph per step (gate, select, gather folded into the layer's RMSNorm, layer)"}


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, w):
    import torch
    from learned_token_pruning_b200 import pipeline, tokengate as tg

    rank, world, dist = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    step = pipeline.GatedPrefillStep(w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    m = step.m

    step.capture()

    def one_step():
        step.replay()

    for _ in range(args.warmup):
        flush.zero_()
        one_step()
    torch.cuda.synchronize(dev)
    tg.tg_check_device_error()

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(visible.split(",")[dev.index]) if visible and visible.split(",")[dev.index].strip().isdigit() \
        else dev.index
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", ""))
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}", gpu_index) if rank == 0 else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter()
    if sampler:
        sampler.start()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        one_step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    wall = time.perf_counter() - t_wall
    clocks = sampler.stop() if sampler else None
    tg.tg_check_device_error()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_s = sum(step_ms) / 1e3
    total_s = max_over_ranks(total_s, dist, dev)
    ms_per_step = total_s * 1e3 / args.steps
    value = replica_value(world, w.n, args.steps, total_s)

    # ---- per-call breakdown (same inputs, each library call bracketed by events on the stream)
    work = workload_work(w, m)
    br = breakdown(step, w, args, stream, flush)
    kernels = {}
    for name, ms in br.items():
        if name.startswith("_"):
            continue
        wk = work.get(name, {})
        entry = {"us": ms * 1e3}
        if ms <= 0:             # serialised replays (under a profiler) can leave no difference to time
            kernels[name] = entry
            continue
        if "flops" in wk and name != "gate_score":
            tf = wk["flops"] / (ms * 1e-3) / 1e12
            entry.update({"tflops": tf, "frac_bf16_peak": tf / peaks["bf16_tflops"]})
        if "bytes" in wk:
            gbs = wk["bytes"] / (ms * 1e-3) / 1e9
            entry.update({"gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]})
        if name == "gate_score":
            # 256 flop per byte of hidden state: its tensor ceiling is as
            # close as its HBM one, so both fractions are given
            entry["tflops"] = wk["flops"] / (ms * 1e-3) / 1e12
            entry["frac_bf16_peak"] = entry["tflops"] / peaks["bf16_tflops"]
        kernels[name] = entry
    # calls timed alone that the step runs fused: tg_gather (folded into the
    # layer's first RMSNorm), tg_gate_score and tg_topk_select (tg_gate_score_select)
    for k in ("unfused_gather", "gate_score", "topk_select"):
        kernels[k]["in_step"] = False
    # what the selector adds inside the fused call (started from the gate's histogram)
    kernels["gate_score_select"]["select_us_beyond_gate"] = kernels["gate_score_select"]["us"] - kernels["gate_score"]["us"]
    not_dom = ("gather_layer_total", "unfused_gather", "gate_score", "topk_select")
    dom = max((k for k in kernels if k not in not_dom and kernels[k]["us"] > 0), key=lambda k: kernels[k]["us"])
    wk = work[dom]
    traffic = measured_traffic(dom, w.n if dom == "gate_score" else m)
    if "flops" in wk and dom != "gate_score":
        roof = {"kernel": dom, "bound": "tensor", "achieved": kernels[dom]["tflops"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": kernels[dom]["tflops"] / peaks["bf16_tflops"], "traffic": traffic, "traffic_unit": "bytes per launch (ncu DRAM read+write)",
                "peak_source": peaks["source"] + " (burst bf16)"}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": kernels[dom]["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": kernels[dom]["gbs"] / peaks["hbm_gbs"], "traffic": traffic, "traffic_unit": "bytes per launch (ncu DRAM read+write)",
                "peak_source": peaks["source"]}

    # ---- end to end through the public API: pinned host inputs in, result back to the host
    e2e = end_to_end(step, w, args, stream, flush, dist, dev, world)

    # gate (with the selector's first-digit histogram), select, gather + RMSNorm,
    # then qkv, q/k-norm + RoPE, attention, o, RMSNorm, gate/up + SwiGLU, down
    launches_per_step = 10
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    # ---- the rest of the metric (single GPU only): the 128K-token step and the
    # 28-layer stack's time to first token at 16K and 128K, pruned and not
    ttft = {"gated_layer_step_n16384": ms_per_step}
    att_frac = {f"n{w.n}_m{m}": kernels["attention"].get("frac_bf16_peak")}
    extras = {}
    if world == 1 and not args.no_extras:
        from learned_token_pruning_b200 import synth
        w128 = synth.long_128k()
        long = single_layer_step(w128, dev, stream, flush, 10, peaks)
        ttft["gated_layer_step_n131072"] = long["step_ms"]
        att_frac[f"n{w128.n}_m{long['kept_rows']}"] = long["attention"]["frac_bf16_peak"]
        extras["long_context_step"] = long
        for n_, k_ in ((16384, 2000), (131072, 8192)):
            r = stack_ttft(n_, k_, [13, 1], 3, dev, stream)
            ttft[f"stack28_n{n_}"] = r
        extras["decode"] = decode_extras(args)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        sec, desc, threads = oracle_step_seconds(w)
        cpu = {"value": w.n / sec, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) hidden, N(0,0.02) weights)",
        "config": config_dict(w, world),
        "ttft_ms": ttft, "attention_frac_bf16_peak": att_frac, **extras,
        "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks, "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def breakdown(step, w, args, stream, flush):
    """Average duration (ms) of each library call of the step, on the step's own inputs."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    D, hq, hkv = w.head_dim, w.hq, w.hkv
    m = step.m
    dt = step.dt
    qkv_w = (hq + 2 * hkv) * D
    # layer intermediates in their own buffers (the layer call keeps them in its workspace)
    xn = torch.randn(m, w.d_model, device=stream.device).to(dt)
    qkv = torch.randn(m, qkv_w, device=stream.device).to(dt)
    att = torch.empty(m, hq * D, dtype=dt, device=stream.device)
    act = torch.empty(m, w.d_ff, dtype=dt, device=stream.device)
    hres = torch.randn(m, w.d_model, device=stream.device).to(dt)
    L = step.layer
    aws_n = tg.attention_workspace_bytes(m, hq, hkv, D, dt)
    aws = torch.empty(max(aws_n, 16), dtype=torch.uint8, device=stream.device) if aws_n else None
    hk_buf = torch.empty_like(step.hidden_kept)
    calls = {
        "gate_score_select": step.gate_select,
        "gate_score": step.gate_score,
        "topk_select": step.select,
        "gather_rmsnorm": lambda: tg.tg_gather_rmsnorm(step.hidden, step.kept, step.scores, step.sumsq,
                                                       step.n_prunable, step.eps_s, L["w_in_norm"], step.norm_eps,
                                                       hk_buf, xn, step.pos, step.bias, step.ratio),
        "attention": lambda: tg.tg_gated_attention(qkv[:, :hq * D], qkv[:, hq * D:(hq + hkv) * D],
                                                   qkv[:, (hq + hkv) * D:], D, step.bias, L["head_gain"],
                                                   L["head_temp"], step.ratio, 1.0 / math.sqrt(D), att,
                                                   ws=aws),
        "linear_qkv": lambda: tg.tg_linear(xn, L["w_qkv"], qkv),
        "linear_o": lambda: tg.tg_linear(att, L["w_o"], hres, tg.TG_EPI_RESIDUAL),
        "linear_gate_up_swiglu": lambda: tg.tg_linear(xn, L["w_gate_up"], act, tg.TG_EPI_SWIGLU),
        "linear_down": lambda: tg.tg_linear(act, L["w_down"], hres, tg.TG_EPI_RESIDUAL),
        "gather_layer_total": step.gather_layer,
        "unfused_gather": step.gather,
    }
    step.run()
    torch.cuda.synchronize()
    reps = max(5, min(args.steps, 50))

    def graph_of(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body()
        return g

    def replay_ms(g):
        # back-to-back replays between one pair of events: the GPU never waits
        # for the host inside the timed interval
        g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # each call is timed as (L2 flush + call) minus (L2 flush): cold L2 like
    # the step, without the flush and without launch gaps.  A call whose input
    # alone is larger than L2 (the gate at 128K tokens reads 512 MiB) finds
    # none of it there anyway; it runs back to back without the flush, whose
    # dirty lines it would otherwise write back to HBM inside its own time.
    l2_bytes = torch.cuda.get_device_properties(stream.device).L2_cache_size
    work = workload_work(w, m)
    g_flush = graph_of(lambda: flush.zero_())
    t_flush = replay_ms(g_flush)
    out = {}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        if work.get(name, {}).get("bytes", 0) > l2_bytes:
            g = graph_of(fn)
            out[name] = replay_ms(g)
            out.setdefault("_unflushed", []).append(name)
        else:
            def body(fn=fn):
                flush.zero_()
                fn()

            g = graph_of(body)
            out[name] = max(replay_ms(g) - t_flush, 0.0)
        del g
    del g_flush
    return out


def end_to_end(step, w, args, stream, flush, dist, dev, world):
    """Same metric through the public API with the inputs in pinned host memory:
    every step copies its hidden states and prunable mask in, runs the four
    calls and copies the kept-row output back, all inside the timed region.
    Steps are pipelined the way a server would run consecutive requests: the
    upload of step i+1 (its own stream, into the other of two device staging
    buffers) overlaps the compute of step i, and the readback of step i (a
    third stream, from the other of two output buffers) overlaps step i+1."""
    import torch
    h_host = step.hidden.cpu().pin_memory()
    m_host = step.prunable.cpu().pin_memory()
    out_host = [torch.empty(step.hidden_kept.shape, dtype=step.hidden_kept.dtype).pin_memory() for _ in range(2)]
    stage_h = [torch.empty_like(step.hidden) for _ in range(2)]
    stage_m = [torch.empty_like(step.prunable) for _ in range(2)]
    stage_o = [torch.empty_like(step.hidden_kept) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    copied, used, computed, read = ([ev() for _ in range(2)] for _ in range(4))
    steps = max(3, min(args.steps, 30))

    def upload(i):
        j = i % 2
        if i >= 2:
            up.wait_event(used[j])          # step i-2 has taken its inputs out of staging buffer j
        with torch.cuda.stream(up):
            stage_h[j].copy_(h_host, non_blocking=True)
            stage_m[j].copy_(m_host, non_blocking=True)
            copied[j].record(up)

    def compute(i):
        j = i % 2
        stream.wait_event(copied[j])
        step.hidden.copy_(stage_h[j], non_blocking=True)
        step.prunable.copy_(stage_m[j], non_blocking=True)
        used[j].record(stream)
        step.replay()
        if i >= 2:
            stream.wait_event(read[j])      # the readback of step i-2 is out of output buffer j
        stage_o[j].copy_(step.hidden_kept, non_blocking=True)
        computed[j].record(stream)

    def readback(i):
        j = i % 2
        down.wait_event(computed[j])
        with torch.cuda.stream(down):
            out_host[j].copy_(stage_o[j], non_blocking=True)
            read[j].record(down)

    def run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
            readback(i)
        stream.wait_event(read[(n - 1) % 2])

    run(3)
    torch.cuda.synchronize()
    barrier(dist, dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    run(steps)
    b.record(stream)
    torch.cuda.synchronize()
    sec = max_over_ranks(a.elapsed_time(b) / 1e3, dist, dev)
    out_ok = torch.equal(out_host[(steps - 1) % 2], step.hidden_kept.cpu())
    return {"value": replica_value(world, w.n, steps, sec), "unit": "tokens/s",
            "h2d_bytes_per_step": h_host.numel() * h_host.element_size() + m_host.numel(),
            "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size(), "steps": steps,
            "pipelined": "upload of step i+1 and readback of step i-1 overlap the compute of step i",
            "readback_matches_device": bool(out_ok)}


def ncu_case():
    """One launch each of the path's kernels, for profiler captures: the fused
    gate score + select at N = 65536 (K = 8192; its input exceeds L2), the
    gather folded into RMSNorm on the 16K-token prefix (K = 2048, 16 question
    tokens), gated attention at m = 2064 and at m = 8256, and the SwiGLU GEMM
    at 2064 rows."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    torch.manual_seed(0)
    dev = "cuda"
    n, d, h, kb = 65536, 2048, 256, 8192
    hid = torch.randn(n, d, device=dev).to(torch.bfloat16)
    w1 = (torch.randn(h, d, device=dev) * 0.02).to(torch.bfloat16)
    w2 = torch.randn(h, device=dev) * 0.02
    mask = torch.ones(n, dtype=torch.uint8, device=dev)
    mask[-64:] = 0
    sc, sq = torch.empty(n, device=dev), torch.empty(1, device=dev)
    ws = torch.empty(tg.tg_workspace_bytes(tg.TG_OP_GATE_SELECT, n=n, d_model=d, h=h), dtype=torch.uint8, device=dev)
    kept64 = torch.empty(kb + 64, dtype=torch.int32, device=dev)
    tg.tg_gate_score_select(hid, None, 1e-6, w1, torch.zeros(h, device=dev), w2, 0.0, mask, n - 64, kb, sc, sq,
                            kept64, ws)
    n16, nq, k = 16384, 16, 2048
    mask16 = torch.ones(n16, dtype=torch.uint8, device=dev)
    mask16[-nq:] = 0
    kept = torch.empty(k + nq, dtype=torch.int32, device=dev)
    tg.tg_topk_select(sc[:n16].contiguous(), mask16, n16 - nq, k, kept)
    hk = torch.empty(k + nq, d, dtype=torch.bfloat16, device=dev)
    xn = torch.empty_like(hk)
    tg.tg_gather_rmsnorm(hid[:n16], kept, sc[:n16].contiguous(), sq, n16 - nq, 1e-6, torch.ones(d, device=dev), 1e-6,
                         hk, xn, torch.empty(k + nq, dtype=torch.int32, device=dev), torch.empty(k + nq, device=dev),
                         torch.empty(k + nq, device=dev))
    hq, hkv, D = 16, 8, 128
    for m in (2064, 8256):
        qkv = torch.randn(m, (hq + 2 * hkv) * D, device=dev).to(torch.bfloat16)
        out = torch.empty(m, hq * D, dtype=torch.bfloat16, device=dev)
        aws_n = tg.attention_workspace_bytes(m, hq, hkv, D, torch.bfloat16)
        aws = torch.empty(max(aws_n, 16), dtype=torch.uint8, device=dev) if aws_n else None
        tg.tg_gated_attention(qkv[:, :hq * D], qkv[:, hq * D:(hq + hkv) * D], qkv[:, (hq + hkv) * D:], D,
                              torch.randn(m, device=dev), torch.rand(hq, device=dev) + 0.5,
                              torch.rand(hq, device=dev) * 0.4 + 0.8, torch.rand(m, device=dev), 1 / math.sqrt(D),
                              out, ws=aws)
    m = 2064
    x = torch.randn(m, 2048, device=dev).to(torch.bfloat16)
    wgu = (torch.randn(2 * 6144, 2048, device=dev) * 0.02).to(torch.bfloat16)
    act = torch.empty(m, 6144, dtype=torch.bfloat16, device=dev)
    tg.tg_linear(x, wgu, act, tg.TG_EPI_SWIGLU)
    torch.cuda.synchronize()
    tg.tg_check_device_error()
    print("ncu case done")


def run_decode(args, emit=None):
    """Decode over the gated KV cache (one new token's attention over the kept
    rows plus the tokens generated so far), per call, L2 flushed before each:
    one record per cache length with the time, the cache bytes read per call
    and their rate against the measured HBM copy bandwidth, printed as a JSON
    line or, with `emit`, passed to it."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    hq, hkv, dh = 16, 8, 128
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for name, m_kept, n_prompt, t in (("qwen3_1.7b_decode_n16384_k2000", 2064, 16384, 64),
                                      ("qwen3_1.7b_decode_n131072_k8192", 8256, 131072, 64),
                                      ("qwen3_1.7b_decode_unpruned_n131072", 131072, 131072, 64)):
        length = m_kept + t + 1
        g = torch.Generator(device=dev).manual_seed(length)
        k = torch.randn(length, hkv * dh, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(length, hkv * dh, device=dev, generator=g).to(torch.bfloat16)
        q = torch.randn(hq, dh, device=dev, generator=g).to(torch.bfloat16)
        bias = torch.randn(length, device=dev, generator=g)
        bias[m_kept:] = 0.0
        gain = torch.rand(hq, device=dev, generator=g) + 0.5
        temp = torch.rand(hq, device=dev, generator=g) * 0.4 + 0.8
        out = torch.empty(hq, dh, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(tg.decode_workspace_bytes(length, hq, hkv, dh), dtype=torch.uint8, device=dev)
        ratio = tg.tg_decode_temperature_ratio(m_kept, n_prompt, t)
        call = lambda: tg.tg_gated_decode_attention(q, k, v, dh, bias, gain, temp, ratio, 1 / math.sqrt(dh), out, ws)
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            call()
        torch.cuda.synchronize(dev)
        reps = max(args.steps, 10)

        def graph_of(body):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                body()
            return gr

        def replay_ms(gr):
            # back-to-back replays between one pair of events on the replaying stream
            gr.replay()
            torch.cuda.synchronize(dev)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                gr.replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) / reps

        def flush_and_call():
            flush.zero_()
            call()

        # (L2 flush + call) minus (L2 flush), as the step's per-call breakdown
        ms = replay_ms(graph_of(flush_and_call)) - replay_ms(graph_of(lambda: flush.zero_()))
        tg.tg_check_device_error()
        nbytes = 2 * length * hkv * dh * 2 + length * 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        rec = {"mode": "decode", "workload": name, "cache_rows": length, "kept_prompt_rows": m_kept,
               "prompt_tokens": n_prompt, "step": t, "us": ms * 1e3, "cache_bytes": nbytes, "gbs": gbs,
               "frac_hbm": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"],
               "l2": "flushed before every call", "ratio": ratio}
        if emit is None:
            print(json.dumps(rec), flush=True)
        else:
            emit(rec)


def decode_extras(args, run=None):
    """Decode over the gated cache for the default JSON line (off the step; the
    same measurement as --decode): per workload its cache rows, time, GB/s and
    HBM fraction.  A failure there leaves {"error": ...} and the line still prints."""
    run = run_decode if run is None else run
    dec = {}
    try:
        run(args, emit=lambda r: dec.__setitem__(r["workload"], {k: r[k] for k in ("cache_rows", "us", "gbs", "frac_hbm")}))
    except Exception as e:
        dec = {"error": f"{type(e).__name__}: {e}"}
    return dec


def run_backward(args):
    """Backward of token-gated attention at the kept rows of the 16K- and
    128K-token prompts (Qwen3-1.7B heads, bf16), per call, L2 flushed before
    each: one JSON line per size with the time, the algorithmic FLOPs (five
    m x m x D contractions per head over the causal half: S, dP, dV, dK, dQ;
    the kernels recompute S and dP once more in the dQ pass, which is not
    counted) and their rate against the measured bf16 tensor peak."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    hq, hkv, dh = 16, 8, 128
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for name, m in (("qwen3_1.7b_attention_backward_k2064", 2064), ("qwen3_1.7b_attention_backward_k8256", 8256)):
        g = torch.Generator(device=dev).manual_seed(m)
        rn = lambda *s: torch.randn(*s, device=dev, generator=g)
        q, k, v, dout = (rn(m, n * dh).to(torch.bfloat16) for n in (hq, hkv, hkv, hq))
        bias, ratio = rn(m), torch.rand(m, device=dev, generator=g) * 0.8 + 0.2
        gain = torch.rand(hq, device=dev, generator=g) + 0.5
        temp = torch.rand(hq, device=dev, generator=g) * 0.4 + 0.8
        out = torch.empty(m, hq * dh, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(hq, m, device=dev)
        scale = 1 / math.sqrt(dh)
        tg.tg_gated_attention(q, k, v, dh, bias, gain, temp, ratio, scale, out, lse)
        dq = torch.empty(m, hq * dh, device=dev)
        dk = torch.empty(m, hkv * dh, device=dev)
        dv = torch.empty(m, hkv * dh, device=dev)
        dbias, dgain, dtemp = torch.empty(m, device=dev), torch.empty(hq, device=dev), torch.empty(hq, device=dev)
        ws = torch.empty(tg.attention_backward_workspace_bytes(m, hq, hkv, dh), dtype=torch.uint8, device=dev)
        call = lambda: tg.tg_gated_attention_backward(q, k, v, out, dout, dh, bias, gain, temp, ratio, scale, lse,
                                                      dq, dk, dv, ws, dbias=dbias, dgain=dgain, dtemp=dtemp)
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            call()
        torch.cuda.synchronize(dev)
        reps = max(min(args.steps, 20), 3)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        total = 0.0
        for _ in range(reps):
            flush.zero_()
            a.record(stream)
            call()
            b.record(stream)
            torch.cuda.synchronize(dev)
            total += a.elapsed_time(b)
        ms = total / reps
        f0.record(stream)
        tg.tg_gated_attention(q, k, v, dh, bias, gain, temp, ratio, scale, out, lse)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        tg.tg_check_device_error()
        flops = 10.0 * dh * hq * m * (m + 1) / 2
        tfs = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"mode": "attention_backward", "workload": name, "rows": m, "hq": hq, "hkv": hkv,
                          "head_dim": dh, "dtype": "bf16 (tensor-core MMAs, fp32 accumulation and gradients)",
                          "us": ms * 1e3, "forward_us": f0.elapsed_time(f1) * 1e3, "flops": flops, "tflops": tfs,
                          "frac_bf16_tensor": tfs / peaks["bf16_tflops"],
                          "peak_source": peaks["source"], "l2": "flushed before every call"}), flush=True)


def ncu_backward_case():
    """One backward call of gated attention at 2064 kept rows (16/8 heads x 128,
    bf16) after a warm-up call, each after an L2 flush, for profiler captures
    of k_attn_bwd_kv_tc and k_attn_bwd_dq_tc."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    dev, hq, hkv, dh, m = "cuda", 16, 8, 128, 2064
    g = torch.Generator(device=dev).manual_seed(2)
    rn = lambda *s: torch.randn(*s, device=dev, generator=g)
    q, k, v, dout = (rn(m, n * dh).to(torch.bfloat16) for n in (hq, hkv, hkv, hq))
    bias, ratio = rn(m), torch.rand(m, device=dev, generator=g) * 0.8 + 0.2
    gain = torch.rand(hq, device=dev, generator=g) + 0.5
    temp = torch.rand(hq, device=dev, generator=g) * 0.4 + 0.8
    out = torch.empty(m, hq * dh, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(hq, m, device=dev)
    scale = 1 / math.sqrt(dh)
    tg.tg_gated_attention(q, k, v, dh, bias, gain, temp, ratio, scale, out, lse)
    dq = torch.empty(m, hq * dh, device=dev)
    dk = torch.empty(m, hkv * dh, device=dev)
    dv = torch.empty(m, hkv * dh, device=dev)
    dbias, dgain, dtemp = torch.empty(m, device=dev), torch.empty(hq, device=dev), torch.empty(hq, device=dev)
    ws = torch.empty(tg.attention_backward_workspace_bytes(m, hq, hkv, dh), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(2):
        flush.zero_()
        tg.tg_gated_attention_backward(q, k, v, out, dout, dh, bias, gain, temp, ratio, scale, lse, dq, dk, dv, ws,
                                       dbias=dbias, dgain=dgain, dtemp=dtemp)
    torch.cuda.synchronize()
    assert tg.tg_check_device_error() == 0


def ncu_decode_case():
    """One decode-attention call on a 131137-row cache (16/8 heads x 128, bf16;
    the unpruned 128K-token prompt's cache) after a warm-up call, each after an
    L2 flush, for profiler captures of the decode kernel (k_decode_tma for a bf16 cache)."""
    import torch
    from learned_token_pruning_b200 import tokengate as tg
    dev, hq, hkv, dh, length = "cuda", 16, 8, 128, 131137
    g = torch.Generator(device=dev).manual_seed(1)
    k = torch.randn(length, hkv * dh, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(length, hkv * dh, device=dev, generator=g).to(torch.bfloat16)
    q = torch.randn(hq, dh, device=dev, generator=g).to(torch.bfloat16)
    bias = torch.randn(length, device=dev, generator=g)
    gain = torch.rand(hq, device=dev, generator=g) + 0.5
    temp = torch.rand(hq, device=dev, generator=g) * 0.4 + 0.8
    out = torch.empty(hq, dh, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(tg.decode_workspace_bytes(length, hq, hkv, dh), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(2):
        flush.zero_()
        tg.tg_gated_decode_attention(q, k, v, dh, bias, gain, temp, 0.9, 1 / math.sqrt(dh), out, ws)
    torch.cuda.synchronize()
    tg.tg_check_device_error()
    print("ncu decode case done")


def run_batch(args):
    """Varlen batching: eight requests of 4K-16K tokens (budget N/8, a 64-token
    question each) through the gated step as one batch (per-request gate,
    select and gather, then one layer call over all kept rows with attention
    per request), against the same eight requests one at a time.  L2 flushed
    before each timed step; one JSON line."""
    import torch
    from learned_token_pruning_b200 import pipeline, synth, tokengate as tg
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    base = synth.qwen3_1p7b_16k()
    lengths = [16384, 8192, 16384, 4096, 12288, 16384, 8192, 4096]
    ws = [dataclasses.replace(base, name=f"req{i}", seed=base.seed + 31 * i, n=n, k=n // 8, plant_len=0)
          for i, n in enumerate(lengths)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 5) if args.steps < 200 else 20

    def timed(replay):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            replay()
        torch.cuda.synchronize(dev)
        total = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            total += a.elapsed_time(b)
        return total / reps

    batch = pipeline.BatchedPrefillStep(ws, dev)
    batch.capture()
    t_batch = timed(batch.replay)
    tg.tg_check_device_error()
    del batch
    torch.cuda.empty_cache()
    singles = [pipeline.GatedPrefillStep(w, dev) for w in ws]
    for st in singles:
        st.capture()
    t_single = timed(lambda: [st.replay() for st in singles])
    tg.tg_check_device_error()
    n_tok = sum(lengths)
    print(json.dumps({"mode": "batch", "workload": "qwen3_1.7b_layer_varlen8_n4k-16k_k_n8",
                      "requests": len(lengths), "tokens": n_tok, "prompt_lengths": lengths,
                      "kept_rows": sum(min(w.k, w.n - w.n_question) + w.n_question for w in ws),
                      "batch_ms": t_batch, "one_at_a_time_ms": t_single,
                      "tokens_per_s_batch": n_tok / (t_batch * 1e-3),
                      "tokens_per_s_one_at_a_time": n_tok / (t_single * 1e-3), "speedup": t_single / t_batch,
                      "l2": "flushed before every timed step", "reps": reps}), flush=True)


def run_sweep(args):
    """The other single-layer workloads (budget sweep at N=32768, K in {1024,
    4096, 8192}; 128K with K=8192): one JSON line each with the step time, the
    per-call breakdown and the peak HBM in use.  Parity cases, not bench lines."""
    import torch
    from learned_token_pruning_b200 import pipeline, synth, tokengate as tg
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for w in [synth.budget_sweep_32k(k) for k in (1024, 4096, 8192)] + [synth.long_128k()]:
        torch.cuda.reset_peak_memory_stats(dev)
        step = pipeline.GatedPrefillStep(w, dev)
        step.capture()
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            step.replay()
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(max(args.steps, 5)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step.replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            times.append(a.elapsed_time(b))
        tg.tg_check_device_error()
        step_ms = sorted(times)[len(times) // 2]
        work = workload_work(w, step.m)
        br = breakdown(step, w, types.SimpleNamespace(steps=max(args.steps, 5)), stream, flush)
        calls = {}
        for name, ms in br.items():
            if name.startswith("_"):
                continue
            e = {"us": round(ms * 1e3, 2)}
            wk = work.get(name, {})
            if "flops" in wk:
                e["tflops"] = round(wk["flops"] / (ms * 1e-3) / 1e12, 1)
                e["frac_bf16_peak"] = round(e["tflops"] / peaks["bf16_tflops"], 3)
            if "bytes" in wk:
                e["gbs"] = round(wk["bytes"] / (ms * 1e-3) / 1e9, 1)
                e["frac_hbm"] = round(e["gbs"] / peaks["hbm_gbs"], 3)
            calls[name] = e
        line = {"mode": "sweep", "workload": w.name, "n": w.n, "k": w.k, "kept_rows": step.m,
                "step_ms": round(step_ms, 4), "tokens_per_s": w.n / (step_ms * 1e-3),
                "peak_hbm_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 3), "calls": calls,
                "l2": "step: flushed before each; calls: flushed before each, except "
                      + (", ".join(br.get("_unflushed", [])) or "none")
                      + " (input larger than L2: back to back, no flush)"}
        print(json.dumps(line), flush=True)
        del step
        torch.cuda.empty_cache()


def stack_ttft(n, k, gate_layers, reps, dev, stream):
    """Time to first token of a random-init 28-layer Qwen3-1.7B-shaped stack
    with the gate at each layer in `gate_layers` (scoring that layer's
    post-attention residual), against the same stack unpruned: from the layer-0
    hidden states in HBM to the last layer's output for the kept rows
    (embedding, final norm and LM head are not part of the path).  Median of
    `reps` runs after one untimed run of each.  Returns a dict."""
    import torch
    from learned_token_pruning_b200 import pipeline, synth, tokengate as tg
    w = synth.full_stack_64k(n=n, k=k, name=f"qwen3_1.7b_stack28_n{n}_k{k}")
    torch.cuda.reset_peak_memory_stats(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    hidden = torch.randn(n, w.d_model, generator=g, device=dev).to(torch.bfloat16)
    prunable = torch.ones(n, dtype=torch.uint8, device=dev)
    prunable[n - w.n_question:] = 0
    gate = {"w1": (torch.randn(w.gate_hidden, w.d_model, generator=g, device=dev) * 0.02).to(torch.bfloat16),
            "b1": torch.zeros(w.gate_hidden, device=dev),
            "w2": torch.randn(w.gate_hidden, generator=g, device=dev) * 0.02, "b2": 0.0}
    layers, heads = pipeline.stack_weights_on_device(w, w.n_layers, dev)
    stacks = {L: pipeline.PrunedPrefillStack(w, hidden, prunable, gate, layers, heads, L) for L in gate_layers}

    def timed(st, fn, reps):
        out = []
        for _ in range(reps):
            st.reset()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            out.append(a.elapsed_time(b))
        return sorted(out)[len(out) // 2]

    st0 = stacks[gate_layers[0]]
    for L, st in stacks.items():
        timed(st, st.run, 1)
    timed(st0, st0.unpruned, 1)
    tg.tg_check_device_error()
    t_full = timed(st0, st0.unpruned, reps)
    res = {"workload": w.name, "n": n, "k": k, "kept_rows": st0.m, "layers": w.n_layers,
           "ttft_unpruned_ms": round(t_full, 3), "reps": reps, "gate": {}}
    for L, st in stacks.items():
        t = timed(st, st.run, reps)
        res["gate"][f"layer{L}"] = {"ttft_ms": round(t, 3), "speedup": round(t_full / t, 3),
                                    "tokens_per_s": n / (t * 1e-3)}
    tg.tg_check_device_error()
    res["peak_hbm_gb"] = round(torch.cuda.max_memory_allocated(dev) / 1e9, 3)
    del stacks, st0, layers, heads, hidden
    torch.cuda.empty_cache()
    return res


def run_stack(args):
    """The 28-layer stack TTFT at N = 16K, 64K and 128K (gate at layer 13, or
    --gate-layer L), pruned against unpruned; one JSON line per N."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    sizes = [(16384, 2000), (65536, 4096), (131072, 8192)]
    if args.stack_n:
        sizes = [x for x in sizes if x[0] in args.stack_n]
    gl = [args.gate_layer] if args.gate_layer is not None else [13]
    for n, k in sizes:
        r = stack_ttft(n, k, gl, max(1, min(args.steps, 3)), dev, stream)
        g = r["gate"][f"layer{gl[0]}"]
        line = {"mode": "stack", "workload": r["workload"], "n": n, "k": k, "kept_rows": r["kept_rows"],
                "layers": r["layers"], "gate_layer": gl[0], "ttft_ms": g["ttft_ms"],
                "ttft_unpruned_ms": r["ttft_unpruned_ms"], "speedup": g["speedup"], "tokens_per_s": g["tokens_per_s"],
                "peak_hbm_gb": r["peak_hbm_gb"],
                "data": "synthetic (seeded on the device: N(0,1) hidden, N(0,0.02) weights)", "reps": r["reps"]}
        print(json.dumps(line), flush=True)


def single_layer_step(w, dev, stream, flush, reps, peaks):
    """Median time of the whole gated step (one CUDA graph, L2 flushed before
    each) on workload w, with the attention call's time and fraction of the
    measured bf16 peak on its kept causal FLOPs."""
    import torch
    from learned_token_pruning_b200 import pipeline, tokengate as tg
    torch.cuda.reset_peak_memory_stats(dev)
    step = pipeline.GatedPrefillStep(w, dev)
    step.capture()
    for _ in range(3):
        flush.zero_()
        step.replay()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b))
    tg.tg_check_device_error()
    ms = sorted(times)[len(times) // 2]
    br = breakdown(step, w, types.SimpleNamespace(steps=reps), stream, flush)
    work = workload_work(w, step.m)
    att_tf = work["attention"]["flops"] / (br["attention"] * 1e-3) / 1e12
    gate_gbs = work["gate_score"]["bytes"] / (br["gate_score"] * 1e-3) / 1e9
    gate_tf = work["gate_score"]["flops"] / (br["gate_score"] * 1e-3) / 1e12
    gs_gbs = work["gate_score_select"]["bytes"] / (br["gate_score_select"] * 1e-3) / 1e9
    res = {"workload": w.name, "n": w.n, "k": w.k, "kept_rows": step.m, "step_ms": round(ms, 4),
           "tokens_per_s": w.n / (ms * 1e-3), "peak_hbm_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 3),
           "attention": {"us": round(br["attention"] * 1e3, 2), "tflops": round(att_tf, 1),
                         "frac_bf16_peak": round(att_tf / peaks["bf16_tflops"], 4)},
           "gate_score": {"us": round(br["gate_score"] * 1e3, 2), "gbs": round(gate_gbs, 1),
                          "frac_hbm": round(gate_gbs / peaks["hbm_gbs"], 4), "tflops": round(gate_tf, 1),
                          "frac_bf16_peak": round(gate_tf / peaks["bf16_tflops"], 4)},
           "gate_score_select": {"us": round(br["gate_score_select"] * 1e3, 2), "gbs": round(gs_gbs, 1),
                                 "frac_hbm": round(gs_gbs / peaks["hbm_gbs"], 4)},
           "topk_select": {"us": round(br["topk_select"] * 1e3, 2)},
           "l2": "step: flushed (256 MiB write) before each; calls: flushed before each, except "
                 + (", ".join(br.get("_unflushed", [])) or "none")
                 + " (input larger than L2: back to back, no flush)",
           "reps": reps}
    del step
    torch.cuda.empty_cache()
    return res


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", action="store_true", help="one launch of each heavy kernel (profiling)")
    ap.add_argument("--sweep", action="store_true", help="budget-sweep and 128K single-layer workloads")
    ap.add_argument("--stack", action="store_true", help="28-layer stack TTFT, pruned vs unpruned")
    ap.add_argument("--decode", action="store_true", help="decode attention over the gated KV cache, per call")
    ap.add_argument("--batch", action="store_true", help="varlen batch of eight requests vs one at a time")
    ap.add_argument("--ncu-decode", action="store_true", help="one decode call on a 131137-row cache (profiling)")
    ap.add_argument("--backward", action="store_true", help="backward of gated attention at the kept-row counts")
    ap.add_argument("--ncu-backward", action="store_true", help="one backward call at 2064 rows (profiling)")
    ap.add_argument("--stack-n", type=int, nargs="*", default=None, help="stack sizes to run (default all)")
    ap.add_argument("--gate-layer", type=int, default=None,
                    help="stack: the layer whose post-attention residual the gate scores (default 13)")
    ap.add_argument("--no-extras", action="store_true",
                    help="default run: skip the 128K step and the 28-layer TTFT figures")
    args = ap.parse_args(argv)
    if args.ncu_case:
        ncu_case()
        return
    if args.ncu_decode:
        ncu_decode_case()
        return
    if args.ncu_backward:
        ncu_backward_case()
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.stack:
        run_stack(args)
        return
    if args.decode:
        run_decode(args)
        return
    if args.batch:
        run_batch(args)
        return
    if args.backward:
        run_backward(args)
        return
    from learned_token_pruning_b200 import synth
    w = synth.qwen3_1p7b_16k()
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
