"""Where the FP8 layer tolerances of tests/test_fp8_gpu.py come from (reading R11 of the DM0.5 page,
section 6.3): one full-width VLM layer with the E4M3 MLP, the oracle's fp32-decision quantiser on
exact operands against the same with the operands perturbed by ~3 fp32 ulps (the GPU forms them in
fp32 in a different order).  A code whose quotient sits within those ulps of an E4M3 midpoint can
round either way, so the comparison is statistical: RMS(d) <= 5e-3, max <= 0.1 and at most 2 % of the
elements beyond 1e-2 of RMS.  Rounding the operands to bf16 before quantising (what the bf16 path feeds
its GEMMs) flips far more codes and breaks those bars, which is why the FP8 path quantises fp32
operands.
"""
import numpy as np
import pytest

from oracle import dm0_oracle as O
from synth import inputs as I


def _stats(got, ref):
    d = np.abs(got - ref)
    r = np.sqrt(np.mean(ref ** 2))
    return float(np.sqrt(np.mean(d ** 2)) / r), float(d.max() / r), float(np.mean(d > 1e-2 * r))


@pytest.fixture(scope="module")
def layer():
    d = I.DM0_BASE.replace(layers=1)
    w = I.Weights(d, seed=0)
    emb = I.prefix_embeddings(d, 1, 128)[0]
    _, _, ref = O.prefill_fp8(w, emb, qrows=O.quantize_rows_f32)
    return d, w, emb, ref


def test_fp32_operand_noise_stays_inside_the_bars(layer):
    d, w, emb, ref = layer
    rng = np.random.default_rng(0)

    def noisy(m):
        m = np.asarray(m, np.float64)
        if not np.array_equal(m, I.round_bf16(m.astype(np.float32))):   # activations, not the bf16 weights
            m = m * (1.0 + 3e-7 * rng.standard_normal(m.shape))
        return O.quantize_rows_f32(m)

    _, _, got = O.prefill_fp8(w, emb, qrows=noisy)
    r_rms, r_max, r_frac = _stats(got, ref)
    print(f"3-ulp noise: RMS {r_rms:.1e} max {r_max:.3f} beyond {r_frac:.4f}")
    assert r_rms <= 5e-3 / 2 and r_max <= 0.1 / 2 and r_frac <= 0.02 / 4


def test_bf16_operands_would_break_them(layer):
    d, w, emb, ref = layer
    _, _, got = O.prefill_fp8(w, emb, qrows=lambda m: O.quantize_rows_f32(I.round_bf16(np.asarray(m, np.float32))))
    r_rms, r_max, r_frac = _stats(got, ref)
    print(f"bf16 operands: RMS {r_rms:.1e} max {r_max:.3f} beyond {r_frac:.4f}")
    assert r_rms > 5e-3 or r_max > 0.1 or r_frac > 0.02
