"""Parity of the FP8 E4M3 prefix-MLP path (reading R11 of the DM0.5 page, section 6.3) with the oracle.

Code decisions are integers decided by floating point, so the oracle side takes them in the GPU
quantiser's precision (quantize_rows_f32: fp32 scale and fp32 quotient).  Tolerances:
  quantiser, same fp32 / bf16 input      bit-exact codes and scales
  quantiser with the pending RMSNorm     scales within 1e-6; at most 0.5 % of codes differ, each by one
                                         E4M3 step (the normalised row is rounded differently in fp32
                                         on the GPU and in fp64 in the oracle)
  FP8 GEMM                               max |d| <= 2e-5 RMS: the products of E4M3 codes are exact in
                                         fp32, only the order of the fp32 summation differs
  FP8 MLP on exact inputs               (a layer whose VLM O-projection is zero, so the MLP's input is the
                                         fp32 input itself) K / V and the action branch as in the bf16
                                         layer test; the VLM output RMS(d) <= 5e-3 RMS, max <= 0.1 RMS and
                                         at most 2 % of the elements beyond 1e-2 RMS: a code whose fp32
                                         quotient lies within a few fp32 ulps of an E4M3 midpoint can round
                                         either way, and one such flip moves a whole output column by a
                                         step of 2^-3 relative (emulated on the CPU with 3-ulp noise on the
                                         operands: max 0.024, RMS 8e-4, 0.2 % of the elements beyond 1e-2)
  FP8 MLP inside the whole layer,        twice the error of the CPU emulation of the GPU's bf16 rounding
  and a whole tiny prefix pass           points followed by the FP8 MLP (tests/tolerances.py): the bf16
                                         rounding of the attention half moves the MLP's input by ~1e-3
                                         relative, and the codes near E4M3 midpoints follow it (measured on
                                         a B200: 1.09e-2 and 1.22e-2 of RMS on the two layers, 2.5e-3 on the
                                         tiny model's layer 1; emulated 1.11e-2, 1.21e-2, 2.4e-3)
"""
import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O
from synth import inputs as I
from tests import tolerances as TOL
from tests.gpu_util import check_bf16, check_fp, host, rel_err, rms, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from vla_dual_expert_b200 import build
    build.build()


def _engine(d, max_batch, max_prefix, w):
    from vla_dual_expert_b200 import Engine
    eng = Engine(d, max_batch, max_prefix)
    eng.load_from(w)
    return eng


@pytest.fixture(scope="module")
def eng1():
    d = I.DM0_BASE.replace(layers=1)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    eng = _engine(d, 2, 816, w)
    yield d, w, eng
    eng.close()


def _decode(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _quant(eng, x, gain=None, ssq=None):
    rows, cols = x.shape
    codes = torch.empty((rows, cols), device="cuda", dtype=torch.uint8)
    scales = torch.empty(rows, device="cuda", dtype=torch.float32)
    eng.op_quant_e4m3(x, codes, scales, gain, ssq)
    eng.sync()
    assert eng.device_error() == 0
    return codes, scales


# ------------------------------------------------------------------ quantiser

@pytest.mark.parametrize("rows,cols", [(3, 8), (37, 2048), (300, 6144)])
def test_quant_bf16_rows_bit_exact(eng1, rows, cols):
    _, _, eng = eng1
    rng = np.random.default_rng(rows)
    x = I.round_bf16((rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-20, 20, (rows, 1)))).astype(np.float32))
    x[rows // 2] = 0.0                                  # all-zero row: scale 1, codes 0
    x[-1, :] = 0.0
    x[-1, cols // 3] = -3.5                             # a single nonzero maps to -448
    codes, scales = _quant(eng, to_dev_bf16(x))
    q, s = O.quantize_rows_f32(x)
    assert np.array_equal(_decode(codes), q)
    assert np.array_equal(host(scales), s[:, 0])


@pytest.mark.parametrize("rows,cols", [(1, 128), (129, 2048)])
def test_quant_f32_rows_bit_exact(eng1, rows, cols):
    _, _, eng = eng1
    rng = np.random.default_rng(100 + rows)
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-8, 8, (rows, 1)))).astype(np.float32)
    codes, scales = _quant(eng, to_dev_f32(x))
    q, s = O.quantize_rows_f32(x)
    assert np.array_equal(_decode(codes), q)
    assert np.array_equal(host(scales), s[:, 0])


def test_quant_with_pending_rmsnorm(eng1):
    d, _, eng = eng1
    rng = np.random.default_rng(7)
    M, H = 200, d.hidden_v
    h = rng.standard_normal((M, H)).astype(np.float32) * 3.0
    g = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    ssq = np.sum(h.astype(np.float64) ** 2, axis=1).astype(np.float32)
    codes, scales = _quant(eng, to_dev_f32(h), to_dev_f32(g), to_dev_f32(ssq))
    r = O.rms_norm(h, g, d.rms_eps)
    q, s = O.quantize_rows_f32(r)
    np.testing.assert_allclose(host(scales), s[:, 0], rtol=1e-6)
    got = _decode(codes)
    differ = got != q
    assert differ.mean() <= 5e-3
    step = np.exp2(np.clip(np.floor(np.log2(np.maximum(np.abs(q[differ]), 2.0 ** -9))), -6, 8) - 3)
    assert np.all(np.abs(got[differ] - q[differ]) <= step * 1.0000001)


# ------------------------------------------------------------------ FP8 GEMM

@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (300, 384, 256), (129, 256, 6144), (816, 12288, 2048)])
def test_gemm_e4m3_matches_exact_products(eng1, M, N, K):
    _, _, eng = eng1
    rng = np.random.default_rng(M + N + K)
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    A, sa = _quant(eng, to_dev_f32(a))
    B, sb = _quant(eng, to_dev_f32(b))
    C = torch.empty((M, N), device="cuda", dtype=torch.float32)
    eng.op_gemm_e4m3(A, sa, B, sb, C)
    eng.sync()
    assert eng.device_error() == 0
    ref = (_decode(A) @ _decode(B).T) * host(sa)[:, None] * host(sb)[None, :]
    check_fp(host(C), ref, 2e-5, f"FP8 GEMM {M}x{N}x{K}")


# ------------------------------------------------------------------ one merged layer with the FP8 VLM MLP

def _fp8_stats(got, ref, what):
    d = np.abs(np.asarray(got, np.float64) - ref)
    r = rms(ref)
    out = (float(np.sqrt(np.mean(d ** 2)) / r), float(d.max() / r), float(np.mean(d > 1e-2 * r)))
    print(f"  {what}: RMS(d)/RMS {out[0]:.2e}  max/RMS {out[1]:.2e}  beyond 1e-2 {out[2]:.2e}")
    return out


def _run_merged(eng, d, B, P, seed, fp8):
    S = d.chunk
    hp = np.stack([I.hidden_states(P, d.hidden_v, seed=seed + b) for b in range(B)])
    hs = np.stack([I.hidden_states(S, d.hidden_a, seed=seed + 100 + b) for b in range(B)])
    outp = torch.empty((B, P, d.hidden_v), device="cuda", dtype=torch.float32)
    outs = torch.empty((B, S, d.hidden_a), device="cuda", dtype=torch.float32)
    k = torch.empty((B, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
    v = torch.empty_like(k)
    eng.set_prefix_fp8(fp8)
    try:
        eng.merged_layer(0, to_dev_f32(hp), to_dev_f32(hs), outp, outs, k, v)
        eng.sync()
    finally:
        eng.set_prefix_fp8(False)
    assert eng.device_error() == 0
    return hp, hs, host(outp), host(outs), host(k), host(v)


@pytest.fixture(scope="module")
def eng_mlp_only():
    """One DM0-base layer whose VLM O-projection is zero: the VLM output is h + MLP(rms(h)), so the FP8
    MLP sees the fp32 input itself and no upstream bf16 rounding."""
    d = I.DM0_BASE.replace(layers=1)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    w.overrides[(0, 0, "Wo")] = np.zeros((d.hidden_v, d.n_q * d.head_dim), np.float32)
    eng = _engine(d, 2, 816, w)
    yield d, w, eng
    eng.close()


@pytest.mark.parametrize("B,P", [(1, 816), (2, 333)])
def test_merged_layer_fp8_mlp(eng_mlp_only, B, P):
    """The FP8 MLP on exact inputs: only fp32 rounding separates the GPU's operands from the oracle's,
    so codes flip only at E4M3 midpoints within a few fp32 ulps (bars of the module docstring)."""
    d, w, eng = eng_mlp_only
    hp, hs, outp, outs, k, v = _run_merged(eng, d, B, P, 40, True)
    for b in range(B):
        rp, rs_, rk, rv = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp[b], hs[b], d, vlm_fp8=O.quantize_rows_f32)
        check_bf16(k[b], rk, TOL.KV_ONE_LAYER[0], "prefix K", TOL.KV_ONE_LAYER[1])
        check_bf16(v[b], rv, TOL.KV_ONE_LAYER[0], "prefix V", TOL.KV_ONE_LAYER[1])
        check_fp(outs[b], rs_, TOL.LAYER, "suffix out (bf16 action branch)")
        r_rms, r_max, r_frac = _fp8_stats(outp[b], rp, "prefix out, FP8 MLP")
        assert r_rms <= 5e-3 and r_max <= 0.1 and r_frac <= 0.02
        # and it is the FP8 MLP that was run: far closer to the FP8 oracle than to the plain one
        plain = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp[b], hs[b], d)[0]
        assert rms(outp[b] - rp) < 0.25 * rms(plain - rp)


@pytest.mark.parametrize("B,P", [(1, 816), (2, 333)])
def test_merged_layer_fp8(eng1, B, P):
    """The whole layer: the MLP's input now carries the bf16 rounding of the attention half (about 1e-3
    relative), and every code within that distance of an E4M3 midpoint may round the other way (a few
    % of them, each by a 2^-3-relative step): the VLM output is held to twice the error the CPU
    emulation of the GPU's rounding points shows on these inputs (tests/tolerances.py FP8_LAYER_RMS),
    and the FP8 path must move the output away from the GPU's own bf16 layer by at least half as much
    as the FP8 oracle moves away from the plain one (the emulation: the same amount)."""
    d, w, eng = eng1
    hp, hs, outp, outs, k, v = _run_merged(eng, d, B, P, 40, True)
    bf = _run_merged(eng, d, B, P, 40, False)[2]
    for b in range(B):
        rp, rs_, rk, rv = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp[b], hs[b], d, vlm_fp8=O.quantize_rows_f32)
        check_bf16(k[b], rk, TOL.KV_ONE_LAYER[0], "prefix K", TOL.KV_ONE_LAYER[1])
        check_fp(outs[b], rs_, TOL.LAYER, "suffix out (bf16 action branch)")
        r_rms, _, _ = _fp8_stats(outp[b], rp, "prefix out, FP8 MLP")
        assert r_rms <= TOL.FP8_LAYER_RMS
        plain = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp[b], hs[b], d)[0]
        assert rms(outp[b] - bf[b]) >= 0.5 * rms(rp - plain)


def test_fp8_toggle_leaves_the_bf16_path_unchanged(eng1):
    """Switching the FP8 MLP on and off again leaves the bf16 layer bit for bit as it was: the VLM path
    has no order-dependent sums (the residual epilogue writes per-group sums of squares that the
    consumer adds in a fixed order)."""
    d, _, eng = eng1
    P, S = 200, d.chunk
    hp, hs = I.hidden_states(P, d.hidden_v, seed=60)[None], I.hidden_states(S, d.hidden_a, seed=61)[None]

    def run():
        outp = torch.empty((1, P, d.hidden_v), device="cuda", dtype=torch.float32)
        outs = torch.empty((1, S, d.hidden_a), device="cuda", dtype=torch.float32)
        k = torch.empty((1, d.n_kv, P, d.head_dim), device="cuda", dtype=torch.bfloat16)
        eng.merged_layer(0, to_dev_f32(hp), to_dev_f32(hs), outp, outs, k, torch.empty_like(k))
        eng.sync()
        return host(outp)

    before = run()
    eng.set_prefix_fp8(True)
    fp8 = run()
    eng.set_prefix_fp8(False)
    after = run()
    assert np.array_equal(after, before)
    assert rel_err(fp8, before) > 1e-3


def test_enable_before_weights_is_a_state_error():
    from vla_dual_expert_b200 import Dm0Error, Engine
    eng = Engine(I.TINY, 1, 64)
    try:
        with pytest.raises(Dm0Error):
            eng.set_prefix_fp8(True)
    finally:
        eng.close()


# ------------------------------------------------------------------ a whole prefix pass (tiny model)

def _tiny_prefill(d, w, emb, fp8):
    from tests.gpu_util import device_view_bf16
    from vla_dual_expert_b200 import Engine
    P = emb.shape[1]
    eng = Engine(d, 1, P)
    try:
        eng.load_from(w)
        eng.set_prefix_fp8(fp8)
        eng.prefill(to_dev_bf16(emb))
        eng.sync()
        assert eng.device_error() == 0
        kp, vp = eng.kv_view()
        K = host(device_view_bf16(kp, (d.layers, d.n_kv, P, d.head_dim)))
        V = host(device_view_bf16(vp, (d.layers, d.n_kv, P, d.head_dim)))
    finally:
        eng.close()
    return K, V


def test_tiny_prefill_fp8():
    """Every layer's K/V after a 2-layer prefix pass with the FP8 MLP: RMS(d) within twice the emulated
    error (tests/tolerances.py FP8_TINY_KV_RMS; layer 0 precedes any MLP), and the FP8 MLP moves layer
    1's K/V away from the GPU's own bf16 prefill by at least half as much as the emulation moves them."""
    from tests import bf16_emulation as E
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    emb = I.prefix_embeddings(d, 1, 64)
    K, V = _tiny_prefill(d, w, emb, True)
    K0, V0 = _tiny_prefill(d, w, emb, False)
    ks, vs, _ = O.prefill_fp8(w, emb[0], qrows=O.quantize_rows_f32)
    eks, evs, _ = E.prefill(w, emb[0], fp8=True)
    eks0, evs0, _ = E.prefill(w, emb[0])
    for l in range(d.layers):
        for got, got0, ref, emu, emu0, nm in ((K[l], K0[l], ks[l], eks[l], eks0[l], "K"),
                                              (V[l], V0[l], vs[l], evs[l], evs0[l], "V")):
            r_rms, _, _ = _fp8_stats(got, ref, f"layer {l} {nm}")
            assert r_rms <= TOL.FP8_TINY_KV_RMS
            if l > 0:
                assert rms(got - got0) >= 0.5 * rms(emu - emu0)
