"""Phase timeline of the single-launch Euler loop (one observation).

With DM0_PERSIST_TRACE=1 set before the context is created, every CTA of the persistent
denoise kernel stamps %globaltimer at fixed points of each phase (see dm0.h, "loop_trace").
`summarize` turns one traced run into per-phase-type medians over the CTAs, in microseconds
from the phase start:

    staged       operand of the phase in shared memory (last staged pair handed to the MMA warp)
    acc_ready    first accumulator segment (GEMM) or first S tile (attention) ready
    issued       results issued (reduce-adds complete / partial O stored)
    arrived      this CTA's grid-barrier arrival
    phase        wall time of the phase (latest start to latest start of the next phase)
    last_arrival latest arrival over the CTAs, from the latest start

    DM0_PERSIST_TRACE=1 python -m vla_dual_expert_b200.loop_trace [--steps K] [--layers L]
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os

import numpy as np

SLOTS = 16
PHASES = ("qkv", "attention", "o_proj", "gate_up", "down")


def read_trace(engine, steps: int) -> np.ndarray:
    """[phases][CTAs][16] timestamps (us, relative to the first start) of the last traced run."""
    import torch
    ptr = ctypes.c_void_p()
    engine._chk(engine.lib.dm0_debug_view(engine.h, b"loop_trace", ctypes.byref(ptr)))
    if not ptr.value:
        raise RuntimeError("no trace: set DM0_PERSIST_TRACE=1 before creating the context")
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    nph = 1 + steps * (5 * engine.dims.layers + 1)
    n = nph * nsm * SLOTS
    view = type("Trace", (), {"__cuda_array_interface__": {"shape": (n,), "typestr": "<u8",
                                                            "data": (ptr.value, False), "version": 3}})()
    arr = torch.as_tensor(view, device="cuda").cpu().numpy().astype(np.float64).reshape(nph, nsm, SLOTS)
    return (arr - arr[0, :, 0].min()) / 1000.0


def summarize(arr: np.ndarray, layers: int, attention_ctas: int) -> dict:
    out: dict = {}
    per_step = 5 * layers + 1
    for q in range(1, arr.shape[0] - 1):
        r = (q - 1) % per_step
        name = "step" if r == 5 * layers else PHASES[r % 5]
        sel = slice(0, attention_ctas) if name == "attention" else slice(None)
        a = arr[q, sel]
        st = a[:, 0]
        rec = {"staged": np.median(a[:, 1] - st), "acc_ready": np.median(a[:, 2] - st),
               "issued": np.median(a[:, 3] - st), "arrived": np.median(a[:, 5] - st),
               "phase": arr[q + 1, :, 0].max() - arr[q, :, 0].max(),
               "last_arrival": arr[q, :, 5].max() - arr[q, :, 0].max()}
        if name == "step":
            rec = {"phase": rec["phase"]}
        out.setdefault(name, []).append(rec)
    return {k: {kk: round(float(np.mean([x[kk] for x in v])), 2) for kk in v[0]} for k, v in out.items()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--layers", type=int, default=28)
    args = ap.parse_args()
    if os.environ.get("DM0_PERSIST_TRACE") != "1":
        raise SystemExit("set DM0_PERSIST_TRACE=1")
    import torch

    from synth import inputs as I
    from vla_dual_expert_b200 import Engine
    d = I.DM0_BASE.replace(layers=args.layers)
    P = 816
    eng = Engine(d, 1, P)
    eng.load_from(I.Weights(d, seed=0))
    n = d.layers * d.n_kv * P * d.head_dim
    g = torch.Generator(device="cuda").manual_seed(3000)
    for ptr in eng.kv_view():
        view = type("Plane", (), {"__cuda_array_interface__": {"shape": (n,), "typestr": "<u2",
                                                                "data": (ptr, False), "version": 3}})()
        torch.as_tensor(view, device="cuda").view(torch.bfloat16).normal_(generator=g)
    eng.kv_commit(1, P)
    noise = torch.from_numpy(I.noise(d, 1)).cuda()
    for _ in range(3):
        eng.denoise(noise, args.steps)
    eng.sync()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    eng.denoise(noise, args.steps)
    ev1.record()
    eng.sync()
    torch.cuda.synchronize()
    arr = read_trace(eng, args.steps)
    splits = 7   # attention items: n_kv x key splits (default 7 splits at P = 816)
    print(json.dumps({"denoise_ms": round(ev0.elapsed_time(ev1), 3), "steps": args.steps, "layers": d.layers,
                      "phases_us": summarize(arr, d.layers, d.n_kv * splits)}, indent=1))
    eng.close()


if __name__ == "__main__":
    main()
