"""Pins of the oracle's FP8 E4M3 prefix-MLP definition (reading R11; the DM0.5 page, section 6.3, names
FP8 E4M3 for the prefix MLP's gate/up/down GEMMs).  Checked against torch's float8_e4m3fn cast (a
library routine) on random values and on every finite code point, hand-worked ties, the error bound
of a 3-bit mantissa, exactness of the scaled GEMM on representable operands, its invariance to
power-of-two input scaling, and the MLP's plumbing against the exact fp64 MLP."""
import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-12, np.log2(448.0), size=20000))   # subnormals to the top binade
    x = mags * rng.choice([-1.0, 1.0], size=mags.size)
    ref = torch.from_numpy(x).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    # the fp32 cast of x can move a value across a tie only if x sits within 2^-24 of it: none here
    assert np.array_equal(O.e4m3(x.astype(np.float32).astype(np.float64)), ref)


def test_every_finite_code_point_is_fixed():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    v = codes.numpy()
    v = v[np.isfinite(v)]
    assert v.size == 254                                   # 256 codes minus the two NaNs
    assert np.array_equal(O.e4m3(v), v)
    assert np.max(v) == O.E4M3_MAX and np.min(v[v > 0]) == 2.0 ** -9


@pytest.mark.parametrize("x,want", [
    (1.0625, 1.0),           # midway 1.0 / 1.125: ties to the even mantissa
    (1.1875, 1.25),          # midway 1.125 / 1.25
    (2.0 ** -10, 0.0),       # half the smallest subnormal: ties to zero
    (3 * 2.0 ** -10, 2.0 ** -8),
    (0.3, 0.3125),
    (448.0, 448.0),
    (464.0, 448.0),          # midway 448 / (480, not a value): ties to even = 448
    (1000.0, 448.0),         # saturates
    (-1000.0, -448.0),
])
def test_hand_worked_roundings(x, want):
    assert O.e4m3(x) == want


def test_relative_error_bound_of_normals():
    rng = np.random.default_rng(12)
    x = np.exp2(rng.uniform(-6, np.log2(448.0), size=50000)) * rng.choice([-1.0, 1.0], size=50000)
    err = np.abs(O.e4m3(x) - x) / np.abs(x)
    assert np.max(err) <= 2.0 ** -4                         # half a unit of the 3-bit mantissa
    assert np.max(err) > 2.0 ** -5                          # and the bound is approached


def test_scaled_gemm_is_exact_on_representable_operands():
    rng = np.random.default_rng(13)
    # integers up to 16 are E4M3 values; a 448 in every row makes each row's scale exactly 1
    x = rng.integers(-16, 17, size=(7, 64)).astype(np.float64)
    w = rng.integers(-16, 17, size=(5, 64)).astype(np.float64)
    x[:, 0], w[:, 0] = 448.0, -448.0
    assert np.array_equal(O.gemm_e4m3(x, w), x @ w.T)


def test_scaled_gemm_commutes_with_power_of_two_scaling():
    rng = np.random.default_rng(14)
    x, w = rng.standard_normal((6, 96)), rng.standard_normal((4, 96))
    base = O.gemm_e4m3(x, w)
    for c in (2.0 ** -7, 0.5, 8.0, 2.0 ** 10):
        assert np.array_equal(O.gemm_e4m3(c * x, w), c * base)
        assert np.array_equal(O.gemm_e4m3(x, c * w), c * base)


def test_quantised_gemm_error_is_bounded():
    rng = np.random.default_rng(15)
    x, w = rng.standard_normal((32, 512)), rng.standard_normal((48, 512))
    exact = x @ w.T
    err = np.sqrt(np.mean((O.gemm_e4m3(x, w) - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert 1e-3 < err < 4e-2


def test_mlp_plumbing_with_an_exact_quantiser():
    rng = np.random.default_rng(16)
    H, I = 64, 96
    w = {"Wg": rng.standard_normal((I, H)) * 0.1, "Wu": rng.standard_normal((I, H)) * 0.1,
         "Wd": rng.standard_normal((H, I)) * 0.1}
    r = rng.standard_normal((10, H))
    exact = (O.silu(r @ w["Wg"].T) * (r @ w["Wu"].T)) @ w["Wd"].T
    got = O.mlp_fp8(w, r, quant=lambda v: v)                # identity: only the scaling remains
    assert np.max(np.abs(got - exact)) <= 1e-12 * np.max(np.abs(exact))
    fp8 = O.mlp_fp8(w, r)
    rel = np.sqrt(np.mean((fp8 - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert 1e-3 < rel < 0.1                                 # E4M3 error, not a wiring error


def test_fp32_quantiser_matches_torch_fp32_arithmetic():
    # the decision in fp32 (the GPU quantiser's precision): torch float32 amax / 448 and float32
    # division, then torch's E4M3 cast (no value exceeds 448 after the division by amax / 448)
    rng = np.random.default_rng(17)
    x = (rng.standard_normal((40, 300)) * np.exp2(rng.uniform(-30, 30, size=(40, 1)))).astype(np.float32)
    x[5] = 0.0
    q, s = O.quantize_rows_f32(x)
    xt = torch.from_numpy(x)
    amax = xt.abs().amax(dim=1, keepdim=True)
    st = torch.where(amax > 0, amax / torch.tensor(448.0, dtype=torch.float32), torch.ones_like(amax))
    ref = (xt / st).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(q, ref) and np.array_equal(s, st.to(torch.float64).numpy())
    assert np.all(np.max(np.abs(q[np.arange(40) != 5]), axis=1) == O.E4M3_MAX)   # the row's amax maps to 448
    assert s[5, 0] == 1.0 and not q[5].any()


def test_fp32_and_fp64_quantisers_differ_only_at_rounding_boundaries():
    # the two decisions agree except where x / s lies within fp32 rounding of an E4M3 midpoint
    rng = np.random.default_rng(18)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    q32, s32 = O.quantize_rows_f32(x)
    q64, s64 = O.quantize_rows(x.astype(np.float64))
    assert np.max(np.abs(s32 / s64 - 1.0)) < 2.0 ** -23
    differ = q32 != q64
    assert differ.mean() < 1e-3
    # where they differ, they are neighbouring E4M3 values (one step apart)
    steps = np.exp2(np.clip(np.floor(np.log2(np.maximum(np.abs(q64[differ]), 2.0 ** -9))), -6, 8) - 3)
    assert np.all(np.abs(q32[differ] - q64[differ]) <= steps * 1.0000001)


def test_fp8_prefill_reduces_to_the_bf16_prefill_with_an_exact_quantiser():
    from synth import inputs as I
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    emb = I.prefix_embeddings(d, 1, 24)[0]
    ks, vs, h = O.prefill(w, emb)
    ident = lambda m: (np.asarray(m, np.float64), np.ones((np.shape(m)[0], 1)))   # noqa: E731
    ks8, vs8, h8 = O.prefill_fp8(w, emb, qrows=ident)
    assert np.max(np.abs(h8 - h)) <= 1e-12 * np.max(np.abs(h))
    for a, b in zip(ks8 + vs8, ks + vs):
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))
    _, _, hq = O.prefill_fp8(w, emb)
    rel = np.sqrt(np.mean((hq - h) ** 2)) / np.sqrt(np.mean(h ** 2))
    assert 1e-5 < rel < 0.05     # E4M3 noise on the MLP branch only, not a wiring error


def test_merged_layer_fp8_switch_touches_only_the_vlm_mlp():
    from synth import inputs as I
    d = I.TINY
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    hp, hs = I.hidden_states(24, d.hidden_v, seed=1), I.hidden_states(d.chunk, d.hidden_a, seed=2)
    ref = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, hs, d)
    ident = lambda m: (np.asarray(m, np.float64), np.ones((np.shape(m)[0], 1)))   # noqa: E731
    same = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, hs, d, vlm_fp8=ident)
    for a, b in zip(same, ref):
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))
    q = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, hs, d, vlm_fp8=True)
    assert np.array_equal(q[1], ref[1]) and np.array_equal(q[2], ref[2]) and np.array_equal(q[3], ref[3])
    assert not np.allclose(q[0], ref[0], rtol=0, atol=1e-6)
