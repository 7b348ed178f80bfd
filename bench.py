#!/usr/bin/env python
"""Throughput of the DM0 merged-attention inference path on B200.

One step = the whole hot path over one batch: dm0_prefill of B prefixes of P
tokens (28 VLM layers, KV cache) + a 10-step Euler dm0_denoise of the
28-layer action expert, producing B action chunks of 50 x 32.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload e2e_b16|e2e_b1]
                    [--impl native|reference]

Default workload e2e_b16: B = 16, P = 2048 (the batched throughput regime);
the same line also carries the batch-1 figure (B = 1, P = 816) under
"batch1".  Inputs are seeded synthetic data of the DM0-base shapes with
random N(0, 0.02) weights.  Multi-GPU: one process per GPU, each rank runs
its own batch (samples are independent: no collective on the data path).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the reference arm of this library).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "action chunks/sec (prefill+10-step denoise) at batch 1 and 16; HBM GB/s, TC util"
EULER_STEPS = 10
# DRAM bytes (read + write) of one prefix-pass gate/up GEMM launch at B=16, P=2048 (M=32768,
# N=12288, K=2048), from an ncu capture of the same kernel and launch shape in `bench.py --one-layer`
# on the current build (n-fastest raster, eight epilogue warps): 0.665 GB read + 0.396 GB written,
# against 0.587 GB algorithmic (activations 134 MB + weights 50 MB read, SwiGLU output 403 MB written);
# the same code measured 0.439 + 0.379 GB on another box
COUNTERS_CURRENT = True
GATEUP_TRAFFIC_BYTES = 1.0602e9
# DRAM bytes (read + write) of the persistent Euler loop per step of 28 action layers at B=1, P=816:
# the ncu capture of `bench.py --b1-loop` (3 layers, 1 step: 104.81 MB read + 3.06 MB written)
# scaled by 28/3; LOOP_COUNTERS_CURRENT is false while the kernel differs from the captured build
LOOP_COUNTERS_CURRENT = True
LOOP_TRAFFIC_BYTES_PER_STEP = 1.0068e9


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self._t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = max(smax, float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax or None, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ algorithmic work per unit

def layer_params(d, branch):
    H, I, D = d.hidden(branch), d.inter(branch), d.head_dim
    return H * (d.n_q + 2 * d.n_kv) * D + d.n_q * D * H + 3 * H * I


def pack_time_mod_weights(weights, d):
    """Blob of the time-modulated expert: the same seeded weights plus the time MLP and modulators."""
    from vla_dual_expert_b200._abi import pack_weights
    return pack_weights(weights, d.layers, time_mod=True)


def prefill_gateup_flops(d, B, P):
    """One VLM gate/up GEMM launch: [B*P x H] x [H -> 2I]."""
    return 2.0 * B * P * d.hidden_v * 2 * d.inter_v


def train_flops(d, B, P):
    """Algorithmic FLOPs of one training step of the action expert: 6 T per parameter (forward, dX,
    dW) for every projection, and 12 S (P + S) D per query head for the merged attention (forward
    Q K^T and P V, adjoint dP, dQ, dK, dV)."""
    T, S = B * d.chunk, d.chunk
    attn = 12.0 * B * d.n_q * S * (P + S) * d.head_dim
    return d.layers * (6.0 * T * layer_params(d, 1) + attn)


def denoise_bytes_per_step(d, B, P):
    """Algorithmic HBM bytes of one Euler step: action-expert bf16 weights + prefix KV cache read once."""
    w = d.layers * layer_params(d, 1) * 2
    kv = d.layers * B * d.n_kv * P * d.head_dim * 2 * 2
    return w + kv


def site_work(d, B, P, name):
    """Algorithmic work of one launch of a probed kernel site: (amount, kind) with kind "flop" (a
    tensor-core contraction) or "byte" (the merged suffix attention, which reads the prefix cache
    once); None for sites without a roofline (the Euler step, the single-launch loop)."""
    D, nq, nkv, S = d.head_dim, d.n_q, d.n_kv, d.chunk
    if "_" not in name:
        return None
    if name.startswith("vlm_"):
        T, H, I = B * P, d.hidden_v, d.inter_v
    else:
        T, H, I = B * S, d.hidden_a, d.inter_a
    site = name.split("_", 1)[1]
    if site == "qkv":
        return 2.0 * T * H * (nq + 2 * nkv) * D, "flop"
    if site == "o":
        return 2.0 * T * nq * D * H, "flop"
    if site == "gateup":
        return 2.0 * T * H * 2 * I, "flop"
    if site == "down":
        return 2.0 * T * I * H, "flop"
    if name == "vlm_attn":
        return 4.0 * B * nq * P * P * D, "flop"
    if name == "act_attn":
        return float(B * nkv * (P + S) * D * 2 * 2), "byte"
    return None


def site_rooflines(d, B, P, bd, peaks):
    """Per-site fraction of its roofline from the probed breakdown (tensor sites against the measured
    sustained bf16 peak, the suffix attention against the measured copy bandwidth)."""
    for name, rec in bd.items():
        w = site_work(d, B, P, name)
        if w is None or not rec["launches"] or rec["avg_us"] <= 0:
            continue
        amount, kind = w
        sec = rec["avg_us"] * 1e-6
        if kind == "flop":
            ach = amount / sec / 1e12
            rec.update({"achieved": round(ach, 1), "unit": "TFLOP/s",
                        "frac": round(ach / peaks["bf16_tflops_sustained"], 4)})
        else:
            ach = amount / sec / 1e9
            rec.update({"achieved": round(ach, 1), "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4)})
    return bd


# ------------------------------------------------------------------ rank plumbing

def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The slowest rank's time (every rank calls this in the same order)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_chunks_per_s(world: int, batch_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank runs its own batch (weak scaling, no cross-rank data)."""
    return world * batch_per_rank * 1000.0 / ms_per_step


# ------------------------------------------------------------------ native arm

def run_native(args, rank, world, local_rank):
    import numpy as np
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))

    def barrier():
        if dist is not None:
            dist.barrier()

    def rank_max(x):
        return max_over_ranks(x, dist, "cuda")

    d = I.DM0_BASE
    wl_main = I.WORKLOADS[args.workload]
    weights = I.Weights(d, seed=0)
    peaks = _peaks()
    eng = Engine(d, max(wl_main.batch, 1), max(wl_main.prefix, 816))
    eng.load_from(weights)
    stream = torch.cuda.current_stream()

    def measure(wl, steps, warmup, probe, eng=eng):
        B, P = wl.batch, wl.prefix
        emb = torch.from_numpy(I.prefix_embeddings(d, B, P, seed=1000 + 97 * rank)).cuda().to(torch.bfloat16)
        noise = torch.from_numpy(I.noise(d, B, seed=2000 + 97 * rank)).cuda()
        out = torch.empty_like(noise)
        for _ in range(warmup):
            eng.prefill(emb)
            eng.denoise(noise, EULER_STEPS, actions=out)
        eng.sync()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        eng.probe(0 if probe is None else 1 << probe)
        launches0 = eng.launch_count()
        with ClockSampler(local_rank) as clk:
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(steps):
                ev[i][0].record(stream)
                eng.prefill(emb)
                ev[i][1].record(stream)
                eng.denoise(noise, EULER_STEPS, actions=out)
                ev[i][2].record(stream)
            t1.record(stream)
            torch.cuda.synchronize()
        barrier()
        launches = eng.launch_count() - launches0
        probe_n, probe_ms = eng.probe_read(probe) if probe is not None else (0, 0.0)
        eng.probe(0)
        eng.sync()
        ms = rank_max(t0.elapsed_time(t1) / steps)
        pre = sorted(e[0].elapsed_time(e[1]) for e in ev)
        den = sorted(e[1].elapsed_time(e[2]) for e in ev)
        assert bool(torch.isfinite(out).all())
        return {"ms": ms, "prefill_ms_p50": pre[len(pre) // 2], "denoise_ms_p50": den[len(den) // 2],
                "prefill_ms_p90": pre[min(len(pre) - 1, int(0.9 * len(pre)))],
                "denoise_ms_p90": den[min(len(den) - 1, int(0.9 * len(den)))],
                "launches": launches, "probe_n": probe_n, "probe_ms": probe_ms, "clocks": clk.summary()}

    def breakdown(eng, wl):
        """One extra (untimed) step with every kernel site probed by CUDA-event pairs: per-site
        milliseconds per step.  Probed launches lose their overlap with the previous kernel and
        the denoise runs without its graph, so the sum exceeds the timed step."""
        from vla_dual_expert_b200 import SITES
        B, P = wl.batch, wl.prefix
        emb = torch.from_numpy(I.prefix_embeddings(d, B, P, seed=1000 + 97 * rank)).cuda().to(torch.bfloat16)
        noise = torch.from_numpy(I.noise(d, B, seed=2000 + 97 * rank)).cuda()
        eng.probe((1 << len(SITES)) - 1)
        eng.prefill(emb)
        eng.denoise(noise, EULER_STEPS)
        eng.sync()
        out = {}
        for i, name in enumerate(SITES):
            n, ms = eng.probe_read(i)
            out[name] = {"launches": n, "ms": round(ms, 3), "avg_us": round(1000.0 * ms / max(n, 1), 2)}
        eng.probe(0)
        return out

    def measure_e2e(wl, steps, warmup):
        """Through dm0_infer_host: pinned host inputs copied in and the chunk copied out every step."""
        B, P = wl.batch, wl.prefix
        emb_bits = torch.from_numpy(I.bf16_bits(I.prefix_embeddings(d, B, P, seed=1000 + 97 * rank)))
        emb_h = torch.empty(emb_bits.shape, dtype=torch.int16, pin_memory=True)
        emb_h.copy_(emb_bits.view(torch.int16))
        noise_h = torch.empty((B, d.chunk, d.action_dim), dtype=torch.float32, pin_memory=True)
        noise_h.copy_(torch.from_numpy(I.noise(d, B, seed=2000 + 97 * rank)))
        out_h = torch.empty_like(noise_h).pin_memory()
        a_emb, a_noise, a_out = emb_h.numpy(), noise_h.numpy(), out_h.numpy()
        for _ in range(warmup):
            eng.infer_host(a_emb, a_noise, EULER_STEPS, actions=a_out)
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            eng.infer_host(a_emb, a_noise, EULER_STEPS, actions=a_out)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = rank_max(t0.elapsed_time(t1) / steps)
        return {"ms": ms, "h2d": emb_h.numel() * 2 + noise_h.numel() * 4, "d2h": out_h.numel() * 4}

    # probe site 3 = the VLM gate/up GEMM of the prefix pass (the largest launch of the step)
    main = measure(wl_main, args.steps, args.warmup, probe=3)
    e2e = measure_e2e(wl_main, max(2, args.steps // 2), 1) if not args.skip_e2e else {"ms": float("nan"), "h2d": 0,
                                                                                        "d2h": 0}
    B, P = wl_main.batch, wl_main.prefix
    value = job_chunks_per_s(world, B, main["ms"])
    gu_ms = main["probe_ms"] / max(main["probe_n"], 1)
    gu_tf = prefill_gateup_flops(d, B, P) / (gu_ms * 1e-3) / 1e12
    tc_peak = peaks["bf16_tflops_sustained"]
    result = {
        "metric": METRIC, "value": round(value, 3), "unit": "chunks/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(main["ms"], 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) prefix embeddings and noise; "
                                                      "random N(0,0.02) DM0-base weights)",
        "config": {"workload": f"{wl_main.name}: prefill B={B} x P={P} + {EULER_STEPS}-step denoise, chunk 50x32, "
                               "DM0-base 28+28 layers", "batch_per_gpu": B, "prefix_len": P,
                   "euler_steps": EULER_STEPS, "parallelism": f"replicas x{world} (data-parallel by sample)",
                   "l2": "inputs larger than L2 (3.7 GB of weights streamed per step)"},
        "prefill_ms_p50": round(main["prefill_ms_p50"], 3), "denoise_ms_p50": round(main["denoise_ms_p50"], 3),
        "prefill_ms_p90": round(main["prefill_ms_p90"], 3), "denoise_ms_p90": round(main["denoise_ms_p90"], 3),
        "roofline": {"bound": "tensor", "kernel": "gemm_tc_persistent<256,4> (prefix-pass gate/up + SwiGLU, M=B*P, N=2*6144, K=2048)",
                     "achieved": round(gu_tf, 1), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(gu_tf / tc_peak, 4),
                     "traffic": GATEUP_TRAFFIC_BYTES if (B, P) == (16, 2048) and COUNTERS_CURRENT else None,
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "peak_src": f"{peaks['src']} bf16_tflops_sustained", "launches": main["probe_n"],
                     "avg_launch_ms": round(gu_ms, 4)},
        "e2e": {"value": (round(job_chunks_per_s(world, B, e2e["ms"]), 3) if e2e["ms"] == e2e["ms"] else None),
                "unit": "chunks/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
        "gpu_launches": main["launches"],
        "clocks": main["clocks"],
    }
    if args.workload == "e2e_b16" and not args.skip_batch1:
        wl1 = I.WORKLOADS["e2e_b1"]
        # at ~18 ms per chunk, 50 chunks give the 200 ms clock sampler a few samples in the timed region
        b1 = measure(wl1, max(args.steps, 50), args.warmup, probe=None)
        den_gbs = denoise_bytes_per_step(d, 1, wl1.prefix) * EULER_STEPS / (b1["denoise_ms_p50"] * 1e-3) / 1e9
        b1_mhz = (b1["clocks"] or {}).get("sm_mhz")
        result["batch1"] = {
            "workload": "e2e_b1: prefill B=1 x P=816 + 10-step denoise",
            "value": round(job_chunks_per_s(world, 1, b1["ms"]), 3),
            "unit": "chunks/s", "ms_per_step": round(b1["ms"], 3), "prefill_ms_p50": round(b1["prefill_ms_p50"], 3),
            "denoise_ms_p50": round(b1["denoise_ms_p50"], 3), "denoise_ms_p90": round(b1["denoise_ms_p90"], 3),
            # the latency-bound loop scales with the SM clock: its time in millions of SM cycles at the
            # median clock sampled during this measurement, comparable across boxes and power states
            "denoise_mcycles_p50": round(b1["denoise_ms_p50"] * b1_mhz / 1000.0, 2) if b1_mhz else None,
            "clocks": b1["clocks"],
            "gpu_launches": b1["launches"],
            "denoise_roofline": {"bound": "hbm",
                                 "kernel": "denoise_persistent_kernel (the 10-step Euler loop, one launch)",
                                 "achieved": round(den_gbs, 1), "peak": peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": round(den_gbs / peaks["hbm_gbs"], 4),
                                 "algorithmic_bytes_per_euler_step": denoise_bytes_per_step(d, 1, wl1.prefix),
                                 "traffic_per_euler_step": LOOP_TRAFFIC_BYTES_PER_STEP if LOOP_COUNTERS_CURRENT else None,
                                 "peak_src": f"{peaks['src']} hbm_gbs"},
        }
    if not args.skip_batch1:
        try:
            result["merged_layer"] = time_merged_layer(eng, d, max(args.steps, 5), args.warmup, stream, rank)
        except Exception as e:   # a side measurement never costs the step's line
            result["merged_layer"] = {"error": str(e)[:200]}
    if args.prefix_fp8:
        # the same step with the VLM MLP's GEMMs in FP8 E4M3 (opt-in; the headline stays bf16): the
        # probed gate/up site covers the operand quantisation and the FP8 GEMM
        eng.set_prefix_fp8(True)
        f8 = measure(wl_main, args.steps, args.warmup, probe=3)
        f8_b1 = measure(I.WORKLOADS["e2e_b1"], max(args.steps, 5), args.warmup, probe=None)
        eng.set_prefix_fp8(False)
        f8_ms = f8["probe_ms"] / max(f8["probe_n"], 1)
        f8_tf = prefill_gateup_flops(d, B, P) / (f8_ms * 1e-3) / 1e12
        fp8_peak = 2.0 * tc_peak
        result["prefix_fp8"] = {
            "value": round(job_chunks_per_s(world, B, f8["ms"]), 3), "unit": "chunks/s",
            "ms_per_step": round(f8["ms"], 3), "prefill_ms_p50": round(f8["prefill_ms_p50"], 3),
            "gateup_site": {"kernels": "quant_rows_e4m3_kernel<float> + gemm_tc_persistent<256,4,true>",
                            "avg_ms": round(f8_ms, 4), "achieved": round(f8_tf, 1), "peak": round(fp8_peak, 1),
                            "unit": "TFLOP/s", "frac": round(f8_tf / fp8_peak, 4),
                            "peak_src": f"{peaks['src']} bf16_tflops_sustained x 2 (nominal fp8 / bf16 ratio)"},
            "gpu_launches": f8["launches"], "clocks": f8["clocks"],
            "batch1": {"value": round(job_chunks_per_s(world, 1, f8_b1["ms"]), 3), "unit": "chunks/s",
                       "prefill_ms_p50": round(f8_b1["prefill_ms_p50"], 3),
                       "denoise_ms_p50": round(f8_b1["denoise_ms_p50"], 3)}}
    if args.train:
        # one flow-matching training step over a prefix cache of the batched workload (opt-in); the
        # single-observation measurements above left a (1, 816) cache, so prefill (B, P) first
        eng.prefill(torch.from_numpy(I.prefix_embeddings(d, B, P, seed=1000 + 97 * rank)).cuda().to(torch.bfloat16))
        a_np, e_np, t_np, m_np = I.train_batch(d, B, seed=4000 + 97 * rank)
        ta, te = torch.from_numpy(a_np).cuda(), torch.from_numpy(e_np).cuda()
        tt = torch.from_numpy(t_np.astype(np.float32)).cuda()
        tm_ = torch.from_numpy(m_np.astype(np.uint8)).cuda()
        grads = torch.empty(eng.grad_floats(), device="cuda", dtype=torch.float32)
        for _ in range(max(1, args.warmup)):
            eng.train_step(ta, te, tt, tm_, grads=grads)
        eng.sync()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        n0 = eng.launch_count()
        t0.record(stream)
        for _ in range(args.steps):
            loss, _ = eng.train_step(ta, te, tt, tm_, grads=grads)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        tms = rank_max(t0.elapsed_time(t1) / args.steps)
        tflop = train_flops(d, B, P) / 1e12
        result["train"] = {"workload": f"flow-matching training step of the 28-layer action expert, B={B} samples of "
                                       f"50x32 over a P={P} prefix cache (knowledge insulation)",
                           "value": round(world * B * 1000.0 / tms, 3), "unit": "samples/s",
                           "ms_per_step": round(tms, 3), "loss": float(loss.item()),
                           "gpu_launches": (eng.launch_count() - n0) // max(args.steps, 1),
                           "roofline": {"bound": "tensor", "algorithmic_tflop_per_step": round(tflop, 3),
                                        "achieved": round(tflop / (tms * 1e-3), 1), "peak": tc_peak,
                                        "unit": "TFLOP/s", "frac": round(tflop / (tms * 1e-3) / tc_peak, 4),
                                        "peak_src": f"{peaks['src']} bf16_tflops_sustained"}}
    if args.time_mod:
        # the same step for the time-modulated action expert (opt-in; its own weights and context)
        from vla_dual_expert_b200 import Engine as _Engine
        eng_tm = _Engine(d, max(wl_main.batch, 1), max(wl_main.prefix, 816), time_mod=True)
        try:
            eng_tm.load_weights(pack_time_mod_weights(weights, d))
            tm = {}
            for wl in (wl_main, I.WORKLOADS["e2e_b1"]):
                r = measure(wl, args.steps, args.warmup, None, eng=eng_tm)
                tm[wl.name] = {"value": round(job_chunks_per_s(world, wl.batch, r["ms"]), 3), "unit": "chunks/s",
                               "ms_per_step": round(r["ms"], 3), "prefill_ms_p50": round(r["prefill_ms_p50"], 3),
                               "denoise_ms_p50": round(r["denoise_ms_p50"], 3), "gpu_launches": r["launches"]}
            result["time_mod"] = tm
        finally:
            eng_tm.close()
    if not args.skip_breakdown:
        result["breakdown_ms_per_step"] = site_rooflines(d, B, P, breakdown(eng, wl_main), peaks)
        if "batch1" in result:
            wl1 = I.WORKLOADS["e2e_b1"]
            result["batch1"]["breakdown_ms_per_step"] = site_rooflines(d, 1, wl1.prefix, breakdown(eng, wl1), peaks)
    if rank == 0 and world == 1 and not args.skip_cpu:
        result["cpu_baseline"] = cpu_baseline(wl_main, budget_s=args.cpu_budget)
        if args.cpu_configs:
            result["cpu_baseline"]["configs_full"] = cpu_configs()
    if rank == 0:
        print(json.dumps(result), flush=True)
    eng.close()
    if dist is not None:
        dist.destroy_process_group()


# ------------------------------------------------------------------ one merged layer

def merged_layer_flops(d, P, S):
    """GEMM and attention FLOPs of one dual-expert layer over [P prefix; S suffix] tokens (B = 1)."""
    gemm = 2 * P * layer_params(d, 0) + 2 * S * layer_params(d, 1)
    D, Hq = d.head_dim, d.n_q
    attn = 4 * Hq * D * (P * P + S * (P + S))   # QK^T and PV: prefix rows see P keys, suffix rows P + S
    return gemm, attn


def time_merged_layer(eng, d, steps, warmup, stream, rank):
    """Microseconds of dm0_merged_layer at full width (one layer, P = 816, S = 50, B = 1)."""
    import torch

    from synth import inputs as I
    P, S = 816, d.chunk
    hp = torch.from_numpy(I.hidden_states(P, d.hidden_v, seed=10 + rank)[None]).cuda()
    hs = torch.from_numpy(I.hidden_states(S, d.hidden_a, seed=110 + rank)[None]).cuda()
    outp, outs = torch.empty_like(hp), torch.empty_like(hs)
    k = torch.empty((1, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for _ in range(warmup):
        eng.merged_layer(0, hp, hs, outp, outs, k, v)
    eng.sync()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        e0.record(stream)
        eng.merged_layer(0, hp, hs, outp, outs, k, v)
        e1.record(stream)
    torch.cuda.synchronize()
    us = sorted(1000.0 * e0.elapsed_time(e1) for e0, e1 in ev)
    p50 = us[len(us) // 2]
    gemm, attn = merged_layer_flops(d, P, S)
    return {"workload": f"one DM0-base merged layer, P={P} prefix + S={S} suffix tokens, B=1",
            "us_p50": round(p50, 1), "us_p90": round(us[min(len(us) - 1, int(0.9 * len(us)))], 1),
            "gemm_gflop": round(gemm / 1e9, 2), "attention_gflop": round(attn / 1e9, 2),
            "achieved_tflops": round((gemm + attn) / (p50 * 1e-6) / 1e12, 1)}


# ------------------------------------------------------------------ the oracle on the host cores

def cpu_baseline(wl, budget_s=20.0):
    """Time the fp64 oracle as it stands on a bounded sample of the workload and scale to chunks/s.

    Sample: VLM layers 0..nv-1 of the prefix pass of sample 0 and na action-expert layer evaluations
    (one Euler step's layers over a prefix cache of length P); the per-chunk time is
    28 * t(VLM layer) + 28 * 10 * t(action layer).
    """
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import dm0_oracle as O
    from synth import inputs as I

    d = wl.dims
    P = wl.prefix
    w = I.Weights(d.replace(layers=2), seed=0)
    emb = I.prefix_embeddings(d, 1, P)[0]
    x = I.noise(d, 1)[0]
    h = np.asarray(emb, np.float64)
    vis = np.ones((P, P), dtype=bool)
    t0 = time.perf_counter()
    nv = 0
    k_last = v_last = None
    while True:
        wv = w.layer(0, nv % 2)
        q, k, v = O.project_qkv(wv, h, np.arange(P), d)
        h = O.finish_layer(wv, h, O.attention(q, k, v, vis), d)
        k_last, v_last = k, v
        nv += 1
        if time.perf_counter() - t0 > budget_s * 0.7 or nv >= 28:
            break
    t_v = (time.perf_counter() - t0) / nv
    head = w.head()
    ha = O.action_input(head, x, 1.0, d)
    t1 = time.perf_counter()
    na = 0
    while True:
        ha = O.suffix_layer(w.layer(1, na % 2), ha, k_last, v_last, d)
        na += 1
        if time.perf_counter() - t1 > budget_s * 0.3 or na >= 280:
            break
    t_a = (time.perf_counter() - t1) / na
    t_chunk = d.layers * t_v + d.layers * EULER_STEPS * t_a
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": round(1.0 / t_chunk, 6), "unit": "chunks/s", "cores": host_cores(), "blas_threads": threads,
            "kind": "oracle", "wall_s": round(time.perf_counter() - t0, 2),
            "sample": f"{nv} VLM layers (P={P}) + {na} action layer evaluations of sample 0, fp64 numpy; "
                      f"per-chunk time extrapolated = 28*{t_v:.3f}s + 280*{t_a:.4f}s"}


def host_cores():
    """Cores this process may run on (the affinity mask, as nproc reports them)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def cpu_configs():
    """The oracle as it stands, timed in full on the host cores on the single-observation configurations:
    one DM0-base merged layer (P = 816, S = 50), the 28-layer 10-step Euler loop over a random 816-token
    cache, and prefill (P = 816) + 10-step denoise.  Wall seconds per configuration."""
    import numpy as np

    from oracle import dm0_oracle as O
    from synth import inputs as I
    d = I.DM0_BASE
    w = I.Weights(d, seed=0)
    out = {"cores": host_cores()}
    hp = I.hidden_states(816, d.hidden_v, seed=10)
    hs = I.hidden_states(d.chunk, d.hidden_a, seed=110)
    w.layer(0, 0), w.layer(1, 0)
    t0 = time.perf_counter()
    O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, hs, d)
    out["merged_layer_s"] = round(time.perf_counter() - t0, 3)
    ks, vs = [], []
    for l in range(d.layers):
        k, v = I.random_kv_layer(d, 1, 816, l)
        ks.append(k[0].astype(np.float64))
        vs.append(v[0].astype(np.float64))
        w.layer(1, l)
    noise = I.noise(d, 1)[0]
    t0 = time.perf_counter()
    O.denoise(w, ks, vs, noise, EULER_STEPS)
    out["denoise_b1_s"] = round(time.perf_counter() - t0, 3)
    emb = I.prefix_embeddings(d, 1, 816)
    for l in range(d.layers):
        w.layer(0, l)
    t0 = time.perf_counter()
    O.infer(w, emb, I.noise(d, 1), EULER_STEPS)
    out["e2e_b1_s"] = round(time.perf_counter() - t0, 3)
    return out


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands on the host cores.  Each step is one bounded sample
    (cpu_baseline) of the workload; ms_per_step is the wall time of a sample step as run, and value is
    the chunks/s the samples extrapolate to (the per-layer times scaled to a whole chunk)."""
    if rank != 0:
        return
    from synth import inputs as I
    wl = I.WORKLOADS[args.workload]
    steps, warmup = max(args.steps, 1), max(args.warmup, 0)
    budget = max(5.0, min(30.0, 150.0 / (steps + warmup)))
    for _ in range(warmup):
        cpu_baseline(wl, budget_s=budget / 3)
    t0 = time.perf_counter()
    vals = [cpu_baseline(wl, budget_s=budget) for _ in range(steps)]
    wall_ms = 1000.0 * (time.perf_counter() - t0) / steps
    v = sum(x["value"] for x in vals) / len(vals)
    cb = dict(vals[-1])
    cb["value"] = round(v, 6)
    res = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "chunks/s", "n_gpus": world,
           "steps": steps, "warmup": warmup, "ms_per_step": round(wall_ms, 1), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "value_basis": "extrapolated: each step times whole VLM layers and action-layer evaluations of one "
                          "sample and scales them to a chunk (28 VLM layers + 280 action layers per sample)",
           "config": {"workload": f"{wl.name}: prefill B={wl.batch} x P={wl.prefix} + {EULER_STEPS}-step denoise "
                                  "(bounded per-layer sample per step, scaled per chunk)"},
           "cpu_baseline": cb, "e2e": {"value": round(v, 6), "unit": "chunks/s", "h2d_bytes_per_step": 0,
                                       "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_one_layer(args):
    """Profiling workload: one DM0-base layer (both experts), by default at B=16, P=2048 — two
    iterations of dm0_prefill + a 1-step dm0_denoise with per-step velocities (direct launches).
    Holds about 2 GB on the device, small enough for full ncu captures of every kernel of the step.
    --batch / --prefix change the shape, --prefix-fp8 runs the VLM MLP in FP8 E4M3, and --train adds
    two flow-matching training steps of the layer after the inference iterations."""
    import numpy as np
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=1)
    B, P = args.batch or 16, args.prefix or 2048
    eng = Engine(d, B, P)
    eng.load_from(I.Weights(d, seed=0))
    if args.prefix_fp8:
        eng.set_prefix_fp8(True)
    emb = torch.from_numpy(I.prefix_embeddings(d, B, P)).cuda().to(torch.bfloat16)
    noise = torch.from_numpy(I.noise(d, B)).cuda()
    vel = torch.empty((1, B, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
    for _ in range(2):
        eng.prefill(emb)
        eng.denoise(noise, 1, velocities=vel)
    out = {"one_layer": "ok", "batch": B, "prefix": P, "prefix_fp8": bool(args.prefix_fp8),
           "mean_abs_velocity": float(vel.abs().mean())}
    if args.train:
        a_np, e_np, t_np, m_np = I.train_batch(d, B, seed=4000)
        ta, te = torch.from_numpy(a_np).cuda(), torch.from_numpy(e_np).cuda()
        tt = torch.from_numpy(t_np.astype(np.float32)).cuda()
        tm_ = torch.from_numpy(m_np.astype(np.uint8)).cuda()
        grads = torch.empty(eng.grad_floats(), device="cuda", dtype=torch.float32)
        for _ in range(2):
            loss, _ = eng.train_step(ta, te, tt, tm_, grads=grads)
        out["train_loss"] = float(loss.item())
    eng.sync()
    print(json.dumps(out))
    eng.close()


def run_b1_loop(args):
    """Profiling workload for the single-launch Euler loop of one observation: DM0-base widths with
    3 action layers (the kernel walks every layer the same way), B=1, a random 816-token prefix cache,
    three 1-step dm0_denoise calls.  Holds about 0.5 GB on the device, small enough for full ncu
    captures of the persistent kernel."""
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=3)
    P = 816
    eng = Engine(d, 1, P)
    eng.load_from(I.Weights(d, seed=0))
    n = d.layers * d.n_kv * P * d.head_dim
    g = torch.Generator(device="cuda").manual_seed(3000)
    for ptr in eng.kv_view():   # the context-owned cache planes, filled in place with N(0, 1)
        view = type("Plane", (), {"__cuda_array_interface__": {"shape": (n,), "typestr": "<u2",
                                                                "data": (ptr, False), "version": 3}})()
        torch.as_tensor(view, device="cuda").view(torch.bfloat16).normal_(generator=g)
    eng.kv_commit(1, P)
    noise = torch.from_numpy(I.noise(d, 1)).cuda()
    n0 = eng.launch_count()
    for _ in range(3):
        out = eng.denoise(noise, 1)
    eng.sync()
    print(json.dumps({"b1_loop": "ok", "launches": eng.launch_count() - n0,
                      "mean_abs_action": float(out.abs().mean())}))
    eng.close()


# ------------------------------------------------------------------ phase timeline of the single-launch loop

# per (phase, CTA) %globaltimer marks of the persistent Euler loop: 0 phase start, 1 operand staged, 2 first
# accumulator (or S tile) ready, 3 results issued, 4 release fence done, 5 barrier arrival, 6 MMA warp saw
# the operand, 7 MMA warp issued its last MMA, 8 operand copies issued, 9 copies landed, 10..15 attention
TRACE_SLOTS = 16
TRACE_PHASES = ("qkv", "attention", "o_proj", "gate_up", "down")


def summarize_loop_trace(arr, layers, items):
    """Per phase type, medians over the CTAs (the attention phase: its first `items` CTAs) and the layer
    passes, in microseconds from the phase's start: staged (operand in shared memory), copies (the operand
    copies in flight), to_copies (from the start until the copies are issued: negative, since the
    barrier's spinning thread issues them before it releases the phase), build (from the copies'
    landing until the operand is staged), acc_ready (first accumulator or S tile), issued (results out), arrived (this CTA's
    barrier arrival); and the phase's wall time (the latest start of the next phase minus its own latest
    start) and last_arrival (the latest arrival minus the latest start).  arr: [rows][CTAs][TRACE_SLOTS]
    ns; row 0 is the first input, then per Euler step 5 rows per layer and one step boundary."""
    import numpy as np
    arr = np.asarray(arr, np.float64) / 1000.0
    per_step = 5 * layers + 1
    acc = {}
    for q in range(1, arr.shape[0] - 1):
        rr = (q - 1) % per_step
        name = "step" if rr == 5 * layers else TRACE_PHASES[rr % 5]
        a = arr[q, :items] if name == "attention" else arr[q]
        st = a[:, 0]
        rec = {"staged": np.median(a[:, 1] - st), "copies": np.median(a[:, 9] - a[:, 8]),
               "to_copies": np.median(a[:, 8] - st), "build": np.median(a[:, 1] - a[:, 9]),
               "acc_ready": np.median(a[:, 2] - st), "issued": np.median(a[:, 3] - st),
               "arrived": np.median(a[:, 5] - st),
               "phase": float(arr[q + 1, :, 0].max() - arr[q, :, 0].max()),
               "last_arrival": float(arr[q, :, 5].max() - arr[q, :, 0].max())}
        if name == "step":
            rec = {"phase": rec["phase"]}
        acc.setdefault(name, []).append(rec)
    return {k: {kk: round(float(np.mean([x[kk] for x in v])), 2) for kk in v[0]} for k, v in acc.items()}


def run_b1_trace(args):
    """Profiling workload: the single-launch Euler loop of one observation at DM0-base widths over a
    random 816-token cache, traced (DM0_PERSIST_TRACE=1 set here before the context is created): every
    CTA stamps %globaltimer at fixed points of each phase.  Prints the loop's CUDA-event time and the
    per-phase medians of summarize_loop_trace."""
    os.environ["DM0_PERSIST_TRACE"] = "1"
    import numpy as np
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=args.trace_layers)
    P, steps = 816, 2
    eng = Engine(d, 1, P)
    eng.load_from(I.Weights(d, seed=0))
    n = d.layers * d.n_kv * P * d.head_dim
    g = torch.Generator(device="cuda").manual_seed(3000)
    for ptr in eng.kv_view():   # the context-owned cache planes, filled in place with N(0, 1)
        view = type("Plane", (), {"__cuda_array_interface__": {"shape": (n,), "typestr": "<u2",
                                                                "data": (ptr, False), "version": 3}})()
        torch.as_tensor(view, device="cuda").view(torch.bfloat16).normal_(generator=g)
    eng.kv_commit(1, P)
    noise = torch.from_numpy(I.noise(d, 1)).cuda()
    for _ in range(3):
        eng.denoise(noise, steps)
    eng.sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    eng.denoise(noise, steps)
    e1.record()
    eng.sync()
    torch.cuda.synchronize()
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    rows = 1 + steps * (5 * d.layers + 1)
    ptr = eng.debug_view("loop_trace")
    view = type("Trace", (), {"__cuda_array_interface__": {"shape": (rows * nsm * TRACE_SLOTS,), "typestr": "<u8",
                                                            "data": (ptr, False), "version": 3}})()
    arr = torch.as_tensor(view, device="cuda").cpu().numpy().reshape(rows, nsm, TRACE_SLOTS)
    arr = arr.astype(np.float64) - float(arr[0, :, 0].min())
    if args.trace_out:
        np.save(args.trace_out, arr)
    splits = min(int(os.environ.get("DM0_PERSIST_SPLITS", "7")), 8)
    nblk = (P + 63) // 64 + 1
    bps = -(-nblk // min(splits, nblk))
    items = d.n_kv * (-(-nblk // bps))
    print(json.dumps({"b1_trace": "ok", "denoise_ms": round(e0.elapsed_time(e1), 3), "steps": steps,
                      "layers": d.layers, "phases_us": summarize_loop_trace(arr, d.layers, items)}))
    eng.close()


GEMM_TRACE_SLOTS = 16
GEMM_TRACE_MARKS = ("entry", "setup", "dep_wait", "first_stage", "first_issued", "first_acc", "first_done",
                    "last_done", "last_load", "exit")


def summarize_gemm_trace(arr):
    """Per launch (rows of `arr`: [launch][CTA][16] %globaltimer marks of the persistent GEMM, CTA 0
    holding the shape in slots 14-15): the shape, the CTAs that ran, the launch span (first entry to
    last exit) and the median over CTAs of each mark after the launch's first entry, in us."""
    import numpy as np
    out = []
    for row in arr:
        m_n, k_bn = int(row[0, 14]), int(row[0, 15])
        if m_n == 0:
            continue
        ran = row[:, 0] > 0
        # CTAs of this launch: their entry is within 1 s of CTA 0's (other rows may be stale)
        ran &= np.abs(row[:, 0].astype(np.float64) - float(row[0, 0])) < 1e9
        r = row[ran].astype(np.float64)
        t0 = r[:, 0].min()
        last = np.maximum(r[:, 6], r[:, 7])   # one-tile CTAs leave "last_done" at 0
        rec = {"M": m_n >> 32, "N": m_n & 0xFFFFFFFF, "K": k_bn >> 32, "BN": k_bn & 0xFFFFFFFF,
               "ctas": int(ran.sum()), "span_us": round((r[:, 9].max() - t0) / 1e3, 2)}
        for i, name in enumerate(GEMM_TRACE_MARKS):
            v = last if name == "last_done" else r[:, i]
            ok = v > 0
            rec[name] = round(float(np.median(v[ok] - t0)) / 1e3, 2) if ok.any() else None
        # QKV epilogue of the CTA's last tile, SM cycles (slots 10-13: group 0 entered, its first head's
        # RMS pass done, that head's RoPE pass done, group 1 done)
        c = r[:, 10:14]
        okc = (c > 0).all(axis=1)
        if okc.any():
            cc = c[okc]
            rec["qkv_epi_kcycles"] = {"rms_pass": round(float(np.median(cc[:, 1] - cc[:, 0])) / 1e3, 2),
                                      "rope_pass": round(float(np.median(cc[:, 2] - cc[:, 1])) / 1e3, 2),
                                      "tile": round(float(np.median(cc[:, 3] - cc[:, 0])) / 1e3, 2)}
        out.append(rec)
    return out


def run_gemm_trace(args):
    """Profiling workload: the one-layer context of --one-layer (--batch / --prefix), with every
    persistent GEMM launch stamping a per-CTA timeline (DM0_GEMM_TRACE=1 set here before the context
    is created).  Two iterations of prefill + a 1-step denoise; prints summarize_gemm_trace of the
    second iteration's launches."""
    os.environ["DM0_GEMM_TRACE"] = "1"
    import numpy as np
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=1)
    B, P = args.batch or 16, args.prefix or 2048
    os.environ["DM0_NO_GRAPH"] = "1"   # direct launches: one trace row per launch
    eng = Engine(d, B, P)
    eng.load_from(I.Weights(d, seed=0))
    emb = torch.from_numpy(I.prefix_embeddings(d, B, P)).cuda().to(torch.bfloat16)
    noise = torch.from_numpy(I.noise(d, B)).cuda()
    for _ in range(2):
        eng.prefill(emb)
        eng.denoise(noise, 1)
    eng.sync()
    torch.cuda.synchronize()
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    rows = 64
    ptr = eng.debug_view("gemm_trace")
    view = type("Trace", (), {"__cuda_array_interface__": {"shape": (rows * nsm * GEMM_TRACE_SLOTS,),
                                                            "typestr": "<u8", "data": (ptr, False), "version": 3}})()
    arr = torch.as_tensor(view, device="cuda").cpu().numpy().reshape(rows, nsm, GEMM_TRACE_SLOTS)
    recs = summarize_gemm_trace(arr)   # launch order
    print(json.dumps({"gemm_trace": "ok", "batch": B, "prefix": P, "launches": recs}))
    eng.close()


def summarize_attn_trace(arr, nblk):
    """Per-block medians over the CTAs of the suffix attention's trace ([CTA][block][4] %globaltimer:
    S seen, max exchanged, P announced, S issued by the MMA warp), in us: the softmax's wait for S
    after announcing the previous P, its S -> max-exchange and max-exchange -> P times, the period
    between consecutive P announcements, and how long before the softmax sees S the MMA warp issued it."""
    import numpy as np
    a = arr[:, :nblk, :].astype(np.float64)
    ok = np.all(a[:, :, :4] > 0, axis=(1, 2))
    a = a[ok]
    if not len(a):   # no CTA of the traced instance ran (small batches use the two-CTAs-per-SM instance)
        return {"ctas": 0, "blocks": nblk}
    med = lambda x: round(float(np.median(x)) / 1e3, 3)   # noqa: E731
    return {"ctas": int(ok.sum()), "blocks": nblk,
            "wait_for_s": med(a[:, 1:, 0] - a[:, :-1, 2]),
            "s_to_max": med(a[:, :, 1] - a[:, :, 0]),
            "max_to_p": med(a[:, :, 2] - a[:, :, 1]),
            "period": med(a[:, 1:, 2] - a[:, :-1, 2]),
            "s_issue_lead": med(a[:, :, 0] - a[:, :, 3]),
            "first_s_seen": med(a[:, 0, 0] - a[:, 0, 3].min()),
            "walk_us": med(a[:, -1, 2] - a[:, 0, 0])}


def run_attn_trace(args):
    """Profiling workload: the one-layer context of --one-layer (B=16, P=2048 by default) with the
    suffix attention stamping %globaltimer per CTA and 64-key block (DM0_ATTN_TRACE=1 set here);
    prints summarize_attn_trace of the last Euler step's launch."""
    os.environ["DM0_ATTN_TRACE"] = "1"
    os.environ["DM0_NO_GRAPH"] = "1"
    import numpy as np
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=1)
    B, P = args.batch or 16, args.prefix or 2048
    eng = Engine(d, B, P)
    eng.load_from(I.Weights(d, seed=0))
    emb = torch.from_numpy(I.prefix_embeddings(d, B, P)).cuda().to(torch.bfloat16)
    noise = torch.from_numpy(I.noise(d, B)).cuda()
    for _ in range(2):
        eng.prefill(emb)
        eng.denoise(noise, 1)
    eng.sync()
    torch.cuda.synchronize()
    ctas = B * d.n_kv
    nblk = (P + 63) // 64 + (d.chunk + 63) // 64
    slots = 1024 * 64 * 4
    ptr = eng.debug_view("attn_trace")
    view = type("Trace", (), {"__cuda_array_interface__": {"shape": (slots,), "typestr": "<u8",
                                                            "data": (ptr, False), "version": 3}})()
    arr = torch.as_tensor(view, device="cuda").cpu().numpy().reshape(1024, 64, 4)[:ctas]
    print(json.dumps({"attn_trace": "ok", "batch": B, "prefix": P,
                      "blocks_us": summarize_attn_trace(arr, min(nblk, 64))}))
    eng.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=("native", "reference"))
    ap.add_argument("--workload", default="e2e_b16", choices=("e2e_b16", "e2e_b1"))
    ap.add_argument("--skip-batch1", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-breakdown", action="store_true")
    ap.add_argument("--one-layer", action="store_true", help="profiling workload: one layer, B=16, P=2048")
    ap.add_argument("--batch", type=int, default=0, help="--one-layer: batch (default 16)")
    ap.add_argument("--prefix", type=int, default=0, help="--one-layer: prefix length (default 2048)")
    ap.add_argument("--b1-loop", action="store_true", help="profiling workload: persistent Euler loop, 3 layers, B=1")
    ap.add_argument("--b1-trace", action="store_true",
                    help="profiling workload: per-phase timeline of the single-launch Euler loop")
    ap.add_argument("--trace-layers", type=int, default=28)
    ap.add_argument("--trace-out", default="", help="--b1-trace: also save the raw [rows][CTAs][slots] ns array (.npy)")
    ap.add_argument("--attn-trace", action="store_true",
                    help="profiling workload: per-block timeline of the merged suffix attention of one layer")
    ap.add_argument("--gemm-trace", action="store_true",
                    help="profiling workload: per-CTA timeline of every persistent GEMM of one layer")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--cpu-configs", action="store_true",
                    help="also time the oracle in full on the single-observation configurations (~1-2 min)")
    ap.add_argument("--train", action="store_true",
                    help="also time one flow-matching training step (reported under train)")
    ap.add_argument("--time-mod", action="store_true",
                    help="also time the step of the time-modulated action expert (reported under time_mod)")
    ap.add_argument("--prefix-fp8", action="store_true",
                    help="also time the step with the VLM MLP in FP8 E4M3 (reported under prefix_fp8)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.one_layer:
        run_one_layer(args)
        return
    if args.b1_loop:
        run_b1_loop(args)
        return
    if args.b1_trace:
        run_b1_trace(args)
        return
    if args.gemm_trace:
        run_gemm_trace(args)
        return
    if args.attn_trace:
        run_attn_trace(args)
        return
    run_native(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
