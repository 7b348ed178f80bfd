"""Pins of the time-modulated action-expert oracle (reading R12 of the DM0.5 page, section 5.2).

Chosen so that a plausible slip fails one of them: the time MLP's layers swapped or its activation
misplaced (closed form from identity weights), the scale/shift/gate order inside a modulator
(stacked identities), a dropped or misplaced gate (all gates zero leaves the residual stream at the
input), a modulated norm that keeps the static gain or drops the shift (scale = -1 makes the final
norm a constant), tau(t) still added to the input (a time-independent condition must make the
velocity time-independent), and the rest of the layer (unit modulation reduces the layer to the
pinned DM0 layer with its static gains, which in turn is pinned by brute force in the DM0 tests).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

from oracle import dm0_oracle as O
from oracle import dm05_oracle as M
from synth import inputs as I

D = I.TINY.replace(layers=2)
P = 16


def _cache(d, seed=3000):
    ks, vs = [], []
    for l in range(d.layers):
        k, v = I.random_kv_layer(d, 1, P, l, seed)
        ks.append(k[0].astype(np.float64))
        vs.append(v[0].astype(np.float64))
    return ks, vs


def _x(d, seed=2000):
    return I.noise(d, 1, seed)[0].astype(np.float64)


def _unit_modulation(w, d, gains):
    """Modulators that reproduce static gains: W = 0, scale bias = gain - 1, shift 0, gate 1."""
    H = d.hidden_a
    for l in range(d.layers):
        lw = w.layer(1, l)
        for name, norm in (("ma", "attn_norm"), ("mm", "mlp_norm")):
            w.overrides[("mod", l, "W_" + name)] = np.zeros((3 * H, H))
            b = np.concatenate([lw[norm] - 1.0, np.zeros(H), np.ones(H)]) if gains else \
                np.concatenate([np.zeros(H), np.zeros(H), np.ones(H)])
            w.overrides[("mod", l, "b_" + name)] = b
    w.overrides[("time", "W_mf")] = np.zeros((2 * H, H))
    w.overrides[("time", "b_mf")] = np.concatenate([w.head()["final_norm"] - 1.0, np.zeros(H)])


def test_time_mlp_closed_form_at_t0():
    # tau(0) = [sin 0 ..., cos 0 ...] = [0]*half + [1]*half; W_ti = 2I, W_to = 3I, no biases:
    # c = 3 silu(2 tau) = [0]*half + [3 silu(2)]*half, silu(2) = 2 / (1 + e^-2)
    H = 8
    d = D.replace(hidden_a=H)
    tw = {"W_ti": 2 * np.eye(H), "b_ti": np.zeros(H), "W_to": 3 * np.eye(H), "b_to": np.zeros(H)}
    c = M.time_condition(tw, 0.0, d)
    silu2 = 2.0 / (1.0 + np.exp(-2.0))
    np.testing.assert_allclose(c, [0.0] * 4 + [3 * silu2] * 4, rtol=1e-15, atol=0)
    # the biases enter before and after the activation: b_ti = -2 cancels the cos half, b_to shifts all
    tw["b_ti"] = np.full(H, -2.0)
    tw["b_to"] = np.full(H, 0.5)
    silu_m2 = -2.0 / (1.0 + np.exp(2.0))
    np.testing.assert_allclose(M.time_condition(tw, 0.0, d), [3 * silu_m2 + 0.5] * 4 + [0.5] * 4,
                               rtol=1e-15, atol=1e-15)


def test_modulation_order_scale_shift_gate():
    H = 6
    c = np.linspace(-2.0, 3.0, H)
    W = np.concatenate([np.eye(H), 2 * np.eye(H), 3 * np.eye(H)])
    b = np.concatenate([np.full(H, 0.1), np.full(H, 0.2), np.full(H, 0.3)])
    g, s, a = M.modulation(W, b, c, 3)
    sc = c / (1.0 + np.exp(-c))
    np.testing.assert_allclose(g, sc + 0.1, rtol=1e-15)
    np.testing.assert_allclose(s, 2 * sc + 0.2, rtol=1e-15)
    np.testing.assert_allclose(a, 3 * sc + 0.3, rtol=1e-15)


def test_ada_rms_matches_torch_rms_norm():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((9, 64))
    g, s = 0.3 * rng.standard_normal(64), rng.standard_normal(64)
    ref = Fnn.rms_norm(torch.tensor(x), (64,), torch.tensor(1.0 + g), eps=1e-6).numpy() + s
    np.testing.assert_allclose(M.ada_rms(x, g, s, 1e-6), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("t", [1.0, 0.3])
def test_unit_modulation_reduces_to_the_dm0_layer(t):
    # DM0 adds tau(t) to the input; with b_in' = b_in + tau(t) the two models see the same input
    w = I.Weights(D, seed=0, gain_jitter=0.1)
    _unit_modulation(w, D, gains=True)
    ks, vs = _cache(D)
    x = _x(D)
    ref = O.velocity(w, ks, vs, x, t)
    w.overrides[("head", "b_in")] = w.head()["b_in"] + O.time_embedding(t, D.hidden_a)
    got = M.velocity(w, ks, vs, x, t)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_zero_gates_leave_the_input_stream():
    w = I.Weights(D, seed=0)
    H = D.hidden_a
    for l in range(D.layers):
        for name in ("ma", "mm"):
            W = np.array(w.mod(l)["W_" + name], np.float64)
            b = np.array(w.mod(l)["b_" + name], np.float64)
            W[2 * H:], b[2 * H:] = 0.0, 0.0
            w.overrides[("mod", l, "W_" + name)] = W
            w.overrides[("mod", l, "b_" + name)] = b
    ks, vs = _cache(D)
    x, t = _x(D), 0.7
    head, tw = w.head(), w.time()
    e = x @ np.asarray(head["W_in"], np.float64).T + head["b_in"]
    c = M.time_condition(tw, t, D)
    mf = np.asarray(tw["W_mf"], np.float64) @ (c / (1.0 + np.exp(-c))) + tw["b_mf"]
    n = e / np.sqrt(np.mean(e * e, axis=-1, keepdims=True) + D.rms_eps)
    ref = (n * (1.0 + mf[:H]) + mf[H:]) @ np.asarray(head["W_out"], np.float64).T + head["b_out"]
    got = M.velocity(w, ks, vs, x, t)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_final_scale_minus_one_makes_the_velocity_constant():
    w = I.Weights(D, seed=0)
    H = D.hidden_a
    shift = np.random.default_rng(6).standard_normal(H)
    w.overrides[("time", "W_mf")] = np.zeros((2 * H, H))
    w.overrides[("time", "b_mf")] = np.concatenate([np.full(H, -1.0), shift])
    ks, vs = _cache(D)
    head = w.head()
    ref = shift @ np.asarray(head["W_out"], np.float64).T + head["b_out"]
    for seed, t in ((2000, 0.9), (2001, 0.1)):
        got = M.velocity(w, ks, vs, _x(D, seed), t)
        assert np.max(np.abs(got - ref[None, :])) <= 1e-12 * np.max(np.abs(ref))


def test_time_enters_only_through_the_condition():
    w = I.Weights(D, seed=0)
    w.overrides[("time", "W_ti")] = np.zeros((D.hidden_a, D.hidden_a))   # c no longer depends on t
    ks, vs = _cache(D)
    x = _x(D)
    assert np.array_equal(M.velocity(w, ks, vs, x, 0.9), M.velocity(w, ks, vs, x, 0.2))
    w2 = I.Weights(D, seed=0)                                            # the default model does
    assert not np.allclose(M.velocity(w2, ks, vs, x, 0.9), M.velocity(w2, ks, vs, x, 0.2))


def test_constant_velocity_euler():
    # W_out = 0: v = b_out exactly, so x_0 = noise - b_out (sum dt = -1)
    w = I.Weights(D, seed=0)
    H = D.hidden_a
    w.overrides[("head", "W_out")] = np.zeros((D.action_dim, H))
    ks, vs = _cache(D)
    x = _x(D)
    x0, vels = M.denoise(w, ks, vs, x, 4)
    np.testing.assert_allclose(x0, x - w.head()["b_out"][None, :], rtol=0, atol=1e-14)
    assert len(vels) == 4
