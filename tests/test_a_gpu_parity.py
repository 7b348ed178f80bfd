"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (tests/tolerances.py), as max |gpu - oracle| / RMS(oracle) unless stated:
  raw GEMM               1e-4  bf16 operands are exact; only the fp32 summation order differs
  one merged layer       1e-2  the stated per-layer bar, fp32 residual-stream outputs of both branches
  action chunk           2e-2  the stated chunk bar; per-step velocities of the 2-layer model too
  bf16-stored tensors    |d_i| <= a * RMS + 2^-8 |ref_i| and RMS(d) <= r * RMS: the 2^-8 term is
                         the rounding of the stored bf16 value itself (2^-9, doubled).
                           K/V cache of one layer        a = 1e-2, r = 5e-3
                           attention output              a = 2e-2, r = 5e-3 (P is also rounded
                                                         to bf16 before PV)
  depth-dependent bars   twice the error of the CPU emulation of the GPU's bf16 rounding points on
                         the same inputs (tests/bf16_emulation.py; tests/test_tolerance_emulation_cpu.py
                         checks them): the K/V of prefill layers 0 / 13 / 27 and of the tiny model, and
                         the velocities at the top of the 28-layer action stack
"""
import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O
from synth import inputs as I
from tests import tolerances as TOL
from tests.gpu_util import check_bf16, check_fp, device_view_bf16, host, rel_err, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

TOL_GEMM, TOL_LAYER, TOL_CHUNK = 1e-4, TOL.LAYER, TOL.CHUNK


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from vla_dual_expert_b200 import build
    build.build()


def _engine(dims, max_batch, max_prefix, weights=None):
    from vla_dual_expert_b200 import Engine
    eng = Engine(dims, max_batch, max_prefix)
    if weights is not None:
        eng.load_from(weights)
    return eng


@pytest.fixture(scope="module")
def layer_engine():
    """DM0-base widths, one layer (head_dim 128): kernel-level tests and the merged layer."""
    d = I.DM0_BASE.replace(layers=1)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    eng = _engine(d, 2, 816, w)
    yield d, w, eng
    eng.close()


# ------------------------------------------------------------------ tensor-core GEMM

@pytest.mark.parametrize("M,N,K", [(300, 384, 192), (128, 512, 1024), (816, 4096, 2048), (50, 256, 64)])
def test_gemm_normal(layer_engine, M, N, K):
    _, _, eng = layer_engine
    rng = np.random.default_rng(M + N + K)
    A = I.round_bf16(rng.standard_normal((M, K)).astype(np.float32))
    B = I.round_bf16(rng.standard_normal((N, K)).astype(np.float32))
    C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.float32)
    eng.op_gemm(to_dev_bf16(A), to_dev_bf16(B), C, swap=0)
    eng.sync()
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    assert rel_err(host(C), ref) <= TOL_GEMM


@pytest.mark.parametrize("M,N,K,splits", [(256, 50, 1024, 1), (256, 50, 1024, 4), (384, 100, 512, 3),
                                          (128, 1, 64, 1), (1024, 64, 3072, 16)])
def test_gemm_swap_split_k(layer_engine, M, N, K, splits):
    _, _, eng = layer_engine
    rng = np.random.default_rng(7 * M + N + K + splits)
    W = I.round_bf16(rng.standard_normal((M, K)).astype(np.float32))
    X = I.round_bf16(rng.standard_normal((N, K)).astype(np.float32))
    C = torch.zeros((N, M), device="cuda", dtype=torch.float32)
    eng.op_gemm(to_dev_bf16(W), to_dev_bf16(X), C, swap=1, splits=splits)
    eng.sync()
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert rel_err(host(C), ref) <= TOL_GEMM


# ------------------------------------------------------------------ merged GQA attention

# the last three launch more than half an SM count of CTAs with suffix keys, which runs the one-CTA-per-SM
# suffix instance (4 K/V stages, two softmax threads per row): an even and an odd number of 64-key
# blocks, and a key split
@pytest.mark.parametrize("B,Tq,Ta,Tb,splits", [(1, 50, 130, 50, 1), (2, 50, 816, 50, 5), (1, 200, 200, 0, 1),
                                               (1, 17, 1, 0, 1), (2, 50, 64, 50, 3), (1, 816, 816, 0, 1),
                                               (2, 800, 816, 50, 1), (2, 400, 640, 37, 1), (2, 800, 816, 50, 2)])
def test_attention(layer_engine, B, Tq, Ta, Tb, splits):
    d, _, eng = layer_engine
    rng = np.random.default_rng(B * 1000 + Tq + Ta + Tb + splits)
    D = d.head_dim
    bf = lambda *s: I.round_bf16(rng.standard_normal(s).astype(np.float32))
    q = bf(B, Tq, d.n_q, D)
    ka, va = bf(B, d.n_kv, Ta, D), bf(B, d.n_kv, Ta, D)
    kb, vb = (bf(B, d.n_kv, Tb, D), bf(B, d.n_kv, Tb, D)) if Tb else (None, None)
    o = torch.full((B, Tq, d.n_q, D), float("nan"), device="cuda", dtype=torch.bfloat16)
    eng.op_attention(to_dev_bf16(q), to_dev_bf16(ka), to_dev_bf16(va), to_dev_bf16(kb) if Tb else None,
                     to_dev_bf16(vb) if Tb else None, o, splits=splits)
    eng.sync()
    for b in range(B):
        k = ka[b] if not Tb else np.concatenate([ka[b], kb[b]], axis=1)
        v = va[b] if not Tb else np.concatenate([va[b], vb[b]], axis=1)
        ref = O.attention(q[b].transpose(1, 0, 2).astype(np.float64), k.astype(np.float64), v.astype(np.float64),
                          np.ones((Tq, Ta + Tb), dtype=bool)).transpose(1, 0, 2)
        check_bf16(host(o[b]), ref, TOL.ATTN_OUT[0], f"attention b={b}", TOL.ATTN_OUT[1])


# ------------------------------------------------------------------ one dual-expert layer

def _check_merged_layer(d, w, eng, layer, B, P, seed):
    S = d.chunk
    hp = np.stack([I.hidden_states(P, d.hidden_v, seed=seed + b) for b in range(B)])
    hs = np.stack([I.hidden_states(S, d.hidden_a, seed=seed + 100 + b) for b in range(B)])
    outp = torch.empty((B, P, d.hidden_v), device="cuda", dtype=torch.float32)
    outs = torch.empty((B, S, d.hidden_a), device="cuda", dtype=torch.float32)
    k = torch.empty((B, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
    v = torch.empty_like(k)
    eng.merged_layer(layer, to_dev_f32(hp), to_dev_f32(hs), outp, outs, k, v)
    eng.sync()
    assert eng.device_error() == 0
    for b in range(B):
        rp, rs, rk, rv = O.merged_layer(w.layer(0, layer), w.layer(1, layer), hp[b], hs[b], d)
        check_fp(host(outp[b]), rp, TOL_LAYER, "prefix out")
        check_fp(host(outs[b]), rs, TOL_LAYER, "suffix out")
        check_bf16(host(k[b]), rk, TOL.KV_ONE_LAYER[0], "prefix K", TOL.KV_ONE_LAYER[1])
        check_bf16(host(v[b]), rv, TOL.KV_ONE_LAYER[0], "prefix V", TOL.KV_ONE_LAYER[1])
        # the layer's own contribution, not only the residual-dominated sum
        assert rel_err(host(outp[b]) - hp[b], rp - hp[b]) <= 3 * TOL_LAYER
        assert rel_err(host(outs[b]) - hs[b], rs - hs[b]) <= 3 * TOL_LAYER


def test_merged_layer_full_width(layer_engine):
    """One DM0-base merged layer, P = 816 (3 x 256 image + 48 text tokens), S = 50, B = 1."""
    d, w, eng = layer_engine
    _check_merged_layer(d, w, eng, 0, 1, 816, seed=10)


def test_merged_layer_full_width_batch2_ragged(layer_engine):
    d, w, eng = layer_engine
    _check_merged_layer(d, w, eng, 0, 2, 333, seed=20)


def test_prefix_outputs_ignore_the_suffix(layer_engine):
    """The block mask on the GPU: prefix rows never attend to suffix keys, so one merged layer's VLM
    output and prefix K/V are bit for bit the same for two different suffixes (the VLM path has no
    order-dependent sums), while the suffix output changes."""
    d, _, eng = layer_engine
    P, S = 816, d.chunk
    hp = I.hidden_states(P, d.hidden_v, seed=50)[None]
    got = []
    for seed in (51, 52):
        hs = I.hidden_states(S, d.hidden_a, seed=seed)[None]
        outp = torch.empty((1, P, d.hidden_v), device="cuda", dtype=torch.float32)
        outs = torch.empty((1, S, d.hidden_a), device="cuda", dtype=torch.float32)
        k = torch.empty((1, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
        v = torch.empty_like(k)
        eng.merged_layer(0, to_dev_f32(hp), to_dev_f32(hs), outp, outs, k, v)
        eng.sync()
        got.append((host(outp), host(k), host(v), host(outs)))
    for i, what in enumerate(("prefix out", "prefix K", "prefix V")):
        assert np.array_equal(got[0][i], got[1][i]), what
    assert rel_err(got[0][3], got[1][3]) > 1e-2


@pytest.mark.parametrize("knob,value", [("DM0_RASTER_BAND", "64"), ("DM0_NO_PDL", "1")])
def test_gemm_schedule_knobs_do_not_change_results(layer_engine, monkeypatch, knob, value):
    """The persistent GEMM's tile order (n-fastest raster or 64-m-tile bands) and programmatic
    dependent launch change only when work runs, never its arithmetic: one merged layer's prefix
    output and K/V (no order-dependent sums on that path) are bit for bit those of the default
    schedule."""
    d, w, eng = layer_engine
    P, S = 816, d.chunk
    hp = to_dev_f32(I.hidden_states(P, d.hidden_v, seed=60)[None])
    hs = to_dev_f32(I.hidden_states(S, d.hidden_a, seed=61)[None])

    def run(e):
        outp = torch.empty((1, P, d.hidden_v), device="cuda", dtype=torch.float32)
        outs = torch.empty((1, S, d.hidden_a), device="cuda", dtype=torch.float32)
        k = torch.empty((1, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
        v = torch.empty_like(k)
        e.merged_layer(0, hp, hs, outp, outs, k, v)
        e.sync()
        assert e.device_error() == 0
        return host(outp), host(k), host(v)

    ref = run(eng)
    monkeypatch.setenv(knob, value)   # read when a context is created
    other = _engine(d, 2, 816, w)
    try:
        got = run(other)
    finally:
        other.close()
    for g, r, what in zip(got, ref, ("prefix out", "prefix K", "prefix V")):
        assert np.array_equal(g, r), what


# ------------------------------------------------------------------ tiny model (2 layers, head_dim 32)

@pytest.fixture(scope="module")
def tiny():
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    eng = _engine(d, 2, 64, w)
    yield d, w, eng
    eng.close()


@pytest.mark.parametrize("B,P", [(1, 64), (2, 37)])
def test_tiny_merged_layer(tiny, B, P):
    d, w, eng = tiny
    _check_merged_layer(d, w, eng, 1, B, P, seed=30)


def _check_stack_velocity(got, ref, what):
    """Velocity at the top of the 28-layer action stack: RMS(d) and max |d| within the emulation-derived
    bars (tests/tolerances.py VEL_STACK: twice the emulated 4.7e-3 and 1.9e-2 of RMS(v))."""
    d = np.abs(np.asarray(got, np.float64) - ref)
    r = float(np.sqrt(np.mean(ref ** 2)))
    rms_e, max_e = float(np.sqrt(np.mean(d ** 2))) / r, float(np.max(d)) / r
    print(f"  {what}: rms err {rms_e:.3e}, max|d|/rms {max_e:.3e}")
    assert rms_e <= TOL.VEL_STACK[0] and max_e <= TOL.VEL_STACK[1], what


def _kv_planes(eng, d, B, P):
    kp, vp = eng.kv_view()
    n = d.layers * B * d.n_kv * P * d.head_dim
    shape = (d.layers, B, d.n_kv, P, d.head_dim)
    return device_view_bf16(kp, (n,)).view(shape), device_view_bf16(vp, (n,)).view(shape)


@pytest.mark.parametrize("B,P,steps", [(1, 64, 4), (2, 37, 3)])
def test_tiny_prefill_and_denoise(tiny, B, P, steps):
    d, w, eng = tiny
    emb = I.prefix_embeddings(d, B, P)
    noise = I.noise(d, B)
    eng.prefill(to_dev_bf16(emb))
    vel = torch.empty((steps, B, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
    chunk = eng.denoise(to_dev_f32(noise), steps, velocities=vel)
    eng.sync()
    kc, vc = _kv_planes(eng, d, B, P)
    ref_chunks, caches, ref_vels = O.infer(w, emb, noise, steps)
    for b in range(B):
        for l in range(d.layers):
            a, r = TOL.KV_TINY
            check_bf16(host(kc[l, b]), caches[b][0][l], a, f"K layer {l}", r)
            check_bf16(host(vc[l, b]), caches[b][1][l], a, f"V layer {l}", r)
        for k in range(steps):
            check_fp(host(vel[k, b]), ref_vels[b][k], TOL_CHUNK, f"velocity step {k}")
    check_fp(host(chunk), ref_chunks, TOL_CHUNK, "chunk")


def test_tiny_graph_replay_matches_direct(tiny):
    """The captured-graph denoise equals the directly launched one (same kernels, same order)."""
    d, w, eng = tiny
    emb, noise = I.prefix_embeddings(d, 1, 64), I.noise(d, 1)
    eng.prefill(to_dev_bf16(emb))
    vel = torch.empty((4, 1, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
    direct = eng.denoise(to_dev_f32(noise), 4, velocities=vel).clone()
    g1 = eng.denoise(to_dev_f32(noise), 4).clone()
    g2 = eng.denoise(to_dev_f32(noise), 4).clone()
    eng.sync()
    ref, _, _ = O.infer(w, emb, noise, 4)
    for got in (direct, g1, g2):
        assert rel_err(host(got), ref) <= TOL_CHUNK
    # atomics make the order of split-K sums vary: runs agree to fp32 noise, not bit for bit
    assert rel_err(host(g1), host(g2)) <= 1e-4


def test_zero_velocity_head_keeps_noise(tiny):
    d, _, _ = tiny
    w = I.Weights(d, seed=2)
    w.overrides[("head", "W_out")] = np.zeros((d.action_dim, d.hidden_a), np.float32)
    w.overrides[("head", "b_out")] = np.zeros(d.action_dim, np.float32)
    eng = _engine(d, 1, 64, w)
    try:
        noise = I.noise(d, 1)
        eng.prefill(to_dev_bf16(I.prefix_embeddings(d, 1, 64)))
        out = eng.denoise(to_dev_f32(noise), 4)
        eng.sync()
        np.testing.assert_array_equal(out.cpu().numpy(), noise)
    finally:
        eng.close()


def test_host_entry_point_matches_device_path(tiny):
    d, w, eng = tiny
    emb, noise = I.prefix_embeddings(d, 2, 40), I.noise(d, 2)
    bits = I.bf16_bits(emb)
    out = eng.infer_host(bits, noise.astype(np.float32), 3)
    ref, _, _ = O.infer(w, emb, noise, 3)
    assert rel_err(out, ref) <= TOL_CHUNK


def test_error_paths(tiny):
    from vla_dual_expert_b200 import Dm0Error
    d, w, _ = tiny
    eng = _engine(d, 1, 64)
    try:
        noise = to_dev_f32(I.noise(d, 1))
        with pytest.raises(Dm0Error) as e:
            eng.denoise(noise, 4)
        assert e.value.status == -6  # no weights
        eng.load_from(w)
        with pytest.raises(Dm0Error) as e:
            eng.denoise(noise, 4)
        assert e.value.status == -6  # no cache
        with pytest.raises(Dm0Error) as e:
            eng.prefill(to_dev_bf16(I.prefix_embeddings(d, 2, 64)))
        assert e.value.status == -2  # B beyond capacity
        eng.prefill(to_dev_bf16(I.prefix_embeddings(d, 1, 64)))
        with pytest.raises(Dm0Error) as e:
            eng.denoise(noise, 0)
        assert e.value.status == -2
        eng.sync()
        assert eng.device_error() == 0
    finally:
        eng.close()


# ------------------------------------------------------------------ full DM0-base model (28 + 28 layers)

@pytest.fixture(scope="module")
def dm0():
    d = I.DM0_BASE
    w = I.Weights(d, seed=0)
    eng = _engine(d, 16, 2048, w)
    yield d, w, eng
    eng.close()


def test_denoise_b1_over_random_prefix_cache(dm0):
    """28-layer action expert, 10 Euler steps, B = 1, over a random N(0,1) bf16 KV cache of 816 tokens."""
    d, w, eng = dm0
    B, P, steps = 1, 816, 10
    kc, vc = _kv_planes(eng, d, B, P)
    ks, vs = [], []
    for l in range(d.layers):
        k, v = I.random_kv_layer(d, B, P, l)
        kc[l].copy_(to_dev_bf16(k))
        vc[l].copy_(to_dev_bf16(v))
        ks.append(k[0].astype(np.float64))
        vs.append(v[0].astype(np.float64))
    eng.kv_commit(B, P)
    noise = I.noise(d, B)
    vel = torch.empty((steps, B, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
    chunk = eng.denoise(to_dev_f32(noise), steps, velocities=vel)
    graphed = eng.denoise(to_dev_f32(noise), steps)
    eng.sync()
    ref, ref_v = O.denoise(w, ks, vs, noise[0], steps)
    for k in range(steps):
        _check_stack_velocity(host(vel[k, 0]), ref_v[k], f"velocity step {k}")
    assert rel_err(host(chunk[0]), ref) <= TOL_CHUNK
    assert rel_err(host(graphed[0]), ref) <= TOL_CHUNK


def test_e2e_b1(dm0):
    """Prefill of 816 prefix tokens + 10-step denoise at batch 1, whole chunk against the oracle."""
    d, w, eng = dm0
    emb, noise = I.prefix_embeddings(d, 1, 816), I.noise(d, 1)
    eng.prefill(to_dev_bf16(emb))
    chunk = eng.denoise(to_dev_f32(noise), 10)
    eng.sync()
    ks, vs, _ = O.prefill(w, emb[0])
    kc, vc = _kv_planes(eng, d, 1, 816)
    for l in (0, 13, 27):
        a, r = TOL.KV_DEPTH_DM0[l]
        check_bf16(host(kc[l, 0]), ks[l], a, f"K layer {l}", r)
        check_bf16(host(vc[l, 0]), vs[l], a, f"V layer {l}", r)
    ref, _ = O.denoise(w, ks, vs, noise[0], 10)
    assert rel_err(host(chunk[0]), ref) <= TOL_CHUNK


def test_e2e_b16_sampled(dm0):
    """Batch 16 x 2048-token prefixes, 10 steps: samples 0 and 15 of the batched run against the oracle."""
    d, w, eng = dm0
    B, P = 16, 2048
    emb, noise = I.prefix_embeddings(d, B, P), I.noise(d, B)
    eng.prefill(to_dev_bf16(emb))
    chunk = eng.denoise(to_dev_f32(noise), 10)
    eng.sync()
    got = host(chunk)
    assert np.all(np.isfinite(got))
    for b in (0, 15):
        ks, vs, _ = O.prefill(w, emb[b])
        ref, _ = O.denoise(w, ks, vs, noise[b], 10)
        assert rel_err(got[b], ref) <= TOL_CHUNK
