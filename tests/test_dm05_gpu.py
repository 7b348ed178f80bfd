"""Parity of the time-modulated action expert (DM0.5 page, section 5.2; reading R12) on the GPU with the
oracle in oracle/dm05_oracle.py.

The modulation tables (every step's scale, shift and gate, and the shifts projected through the QKV
and gate/up weights) are built once per Euler loop from bf16 operands, and the layers then run the
DM0 kernels with a feature bias, a gate and per-step gains, so the DM0 tolerances apply: the final
chunk within 2e-2 of RMS and each step's velocity within 2e-2 of RMS(v) (max), against the oracle's
fp64 definition.  Measured on a B200: chunks and velocities within 3.8e-3 of RMS.
"""
import os

import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O
from oracle import dm05_oracle as M
from synth import inputs as I
from tests.gpu_util import check_fp, host, to_dev_bf16

pytestmark = pytest.mark.gpu

TOL_CHUNK = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from vla_dual_expert_b200 import build
    build.build()


def _engine(d, B, P, w):
    from vla_dual_expert_b200 import Engine
    eng = Engine(d, B, P, time_mod=True)
    eng.load_from(w)
    return eng


def _check(got_x, got_v, ref_x, ref_v, what):
    check_fp(got_x, ref_x, TOL_CHUNK, f"{what}: chunk")
    for k, (gv, rv) in enumerate(zip(got_v, ref_v)):
        check_fp(gv, rv, TOL_CHUNK, f"{what}: velocity of step {k}")


@pytest.mark.parametrize("B,P,steps", [(1, 64, 4), (2, 37, 3)])
def test_tiny_time_modulated_prefill_and_denoise(B, P, steps):
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    emb, noise = I.prefix_embeddings(d, B, P), I.noise(d, B)
    eng = _engine(d, B, P, w)
    try:
        eng.prefill(to_dev_bf16(emb))
        vel = torch.empty((steps, B, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
        out = eng.denoise(torch.from_numpy(noise).cuda(), steps, velocities=vel)
        eng.sync()
        assert eng.device_error() == 0
        x, v = host(out), host(vel)
    finally:
        eng.close()
    for b in range(B):
        ks, vs, _ = O.prefill(w, emb[b])
        rx, rv = M.denoise(w, ks, vs, noise[b], steps)
        _check(x[b], [v[k, b] for k in range(steps)], rx, rv, f"tiny b={b}")


def test_full_width_two_layers_over_a_random_cache():
    """DM0-base widths (head_dim 128), 2 layers, a random 100-token prefix cache, B = 2, 3 steps,
    through the CUDA graph (no velocities requested) and directly (velocities requested)."""
    d = I.DM0_BASE.replace(layers=2)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    B, P, steps = 2, 100, 3
    eng = _engine(d, B, P, w)
    try:
        kp, vp = eng.kv_view()
        from tests.gpu_util import device_view_bf16
        K = device_view_bf16(kp, (d.layers, B, d.n_kv, P, d.head_dim))
        V = device_view_bf16(vp, (d.layers, B, d.n_kv, P, d.head_dim))
        caches = [([], []) for _ in range(B)]
        for l in range(d.layers):
            k, v = I.random_kv_layer(d, B, P, l)
            K[l].copy_(to_dev_bf16(k))
            V[l].copy_(to_dev_bf16(v))
            for b in range(B):
                caches[b][0].append(k[b].astype(np.float64))
                caches[b][1].append(v[b].astype(np.float64))
        eng.kv_commit(B, P)
        noise = I.noise(d, B)
        x_graph = host(eng.denoise(torch.from_numpy(noise).cuda(), steps))
        vel = torch.empty((steps, B, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
        x_direct = host(eng.denoise(torch.from_numpy(noise).cuda(), steps, velocities=vel))
        eng.sync()
        assert eng.device_error() == 0
        v = host(vel)
    finally:
        eng.close()
    for b in range(B):
        rx, rv = M.denoise(w, caches[b][0], caches[b][1], noise[b], steps)
        _check(x_direct[b], [v[k, b] for k in range(steps)], rx, rv, f"base b={b}")
        check_fp(x_graph[b], rx, TOL_CHUNK, f"base b={b}: chunk through the graph")


def test_zero_velocity_head_keeps_noise():
    """W_out = 0 and b_out = 0: every velocity is exactly 0 whatever the modulation, so x_0 = noise."""
    d = I.TINY
    w = I.Weights(d, seed=0)
    w.overrides[("head", "W_out")] = np.zeros((d.action_dim, d.hidden_a), np.float32)
    w.overrides[("head", "b_out")] = np.zeros(d.action_dim, np.float32)
    eng = _engine(d, 1, 64, w)
    try:
        eng.prefill(to_dev_bf16(I.prefix_embeddings(d, 1, 64)))
        noise = I.noise(d, 1)
        x = host(eng.denoise(torch.from_numpy(noise).cuda(), 5))
        eng.sync()
    finally:
        eng.close()
    assert np.array_equal(x, noise.astype(np.float64))


def test_single_observation_runs_as_one_persistent_launch():
    """DM0-base widths, B = 1: the time-modulated Euler loop is the persistent kernel's modulated
    instantiation (one launch after the table pass), against the oracle and against the per-layer
    kernels of the same inputs."""
    d = I.DM0_BASE.replace(layers=2)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    P, steps = 100, 3
    noise = I.noise(d, 1)
    k_np, v_np = zip(*[I.random_kv_layer(d, 1, P, l) for l in range(d.layers)])
    results = {}
    for mode in ("persistent", "per_layer"):
        if mode == "per_layer":
            os.environ["DM0_NO_PERSIST"] = "1"
        try:
            eng = _engine(d, 1, P, w)
        finally:
            os.environ.pop("DM0_NO_PERSIST", None)
        try:
            from tests.gpu_util import device_view_bf16
            kp, vp = eng.kv_view()
            K = device_view_bf16(kp, (d.layers, 1, d.n_kv, P, d.head_dim))
            V = device_view_bf16(vp, (d.layers, 1, d.n_kv, P, d.head_dim))
            for l in range(d.layers):
                K[l].copy_(to_dev_bf16(k_np[l]))
                V[l].copy_(to_dev_bf16(v_np[l]))
            eng.kv_commit(1, P)
            n0 = eng.launch_count()
            x = host(eng.denoise(torch.from_numpy(noise).cuda(), steps))
            eng.sync()
            assert eng.device_error() == 0
            results[mode] = (x, eng.launch_count() - n0)
        finally:
            eng.close()
    ks = [k[0].astype(np.float64) for k in k_np]
    vs = [v[0].astype(np.float64) for v in v_np]
    rx, _ = M.denoise(w, ks, vs, noise[0], steps)
    check_fp(results["persistent"][0][0], rx, TOL_CHUNK, "persistent chunk")
    check_fp(results["persistent"][0][0], results["per_layer"][0][0], 1e-2, "persistent vs per-layer")
    assert results["persistent"][1] < results["per_layer"][1]


def test_modulation_tables_match_the_oracle():
    """The per-loop tables (what every layer of every step reads) against the oracle's time condition
    and modulators: rows within bf16-operand accuracy of modulation(W, b, c(t_k)), scales stored as
    1 + scale, and the QKV shift bias equal to W_qkv bf16(shift)."""
    from tests.gpu_util import _Cai
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    steps, P = 4, 16
    eng = _engine(d, 1, P, w)
    try:
        eng.prefill(to_dev_bf16(I.prefix_embeddings(d, 1, P)))
        eng.denoise(torch.from_numpy(I.noise(d, 1)).cuda(), steps)
        eng.sync()
        H, L = d.hidden_a, d.layers
        R = (6 * L + 2) * H
        QR = (d.n_q + 2 * d.n_kv) * d.head_dim
        mod = torch.as_tensor(_Cai(eng.debug_view("tm_mod"), (steps, R), "<f4"), device="cuda").cpu().numpy()
        bqkv = torch.as_tensor(_Cai(eng.debug_view("tm_bqkv"), (L, steps, QR), "<f4"), device="cuda").cpu().numpy()
    finally:
        eng.close()
    for k, t in enumerate(O.euler_times(steps)):
        c = M.time_condition(w.time(), t, d)
        for l in range(L):
            m = w.mod(l)
            ga, sa, aa = M.modulation(m["W_ma"], m["b_ma"], c, 3)
            gm, sm, am = M.modulation(m["W_mm"], m["b_mm"], c, 3)
            row = mod[k, 6 * l * H:6 * (l + 1) * H]
            ref = np.concatenate([1 + ga, sa, aa, 1 + gm, sm, am])
            assert np.max(np.abs(row - ref)) <= 2e-2 * np.max(np.abs(ref)), (k, l)
            lw = w.layer(1, l)
            wqkv = np.concatenate([lw["Wq"], lw["Wk"], lw["Wv"]]).astype(np.float64)
            shift = I.round_bf16(row[H:2 * H].astype(np.float32)).astype(np.float64)
            np.testing.assert_allclose(bqkv[l, k], wqkv @ shift, rtol=0, atol=1e-4 * np.max(np.abs(wqkv @ shift)))
        gf, sf = M.modulation(w.time()["W_mf"], w.time()["b_mf"], c, 2)
        fin = mod[k, 6 * L * H:]
        assert np.max(np.abs(fin - np.concatenate([1 + gf, sf]))) <= 2e-2 * np.max(np.abs(np.concatenate([1 + gf, sf])))
