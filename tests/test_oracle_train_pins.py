"""Pins of the flow-matching training-step oracle (reading R13 of the DM0.5 page, section 5.3, and the
knowledge-insulation remark of the DM0 architecture notes, section 1).

The hand-written backward is checked against central finite differences of the loss computed through
the DM0 oracle's forward (itself pinned by brute force and library routines), one random direction
per parameter tensor, so a dropped term, a wrong sign or a transposed operand in any adjoint fails
the tensor it feeds.  The loss is pinned by the page's definition of x_t / u_t at its end points, by
a closed form when the velocity is a constant, by its normalisation over the valid entries of the
whole batch, and by the mask.
"""
import numpy as np
import pytest

from oracle import dm0_oracle as O
from oracle import dm0_train as T
from synth import inputs as I

D = I.TINY.replace(layers=2)
P = 16


def _caches(d, B, seed=3000):
    out = []
    for b in range(B):
        ks, vs = [], []
        for l in range(d.layers):
            k, v = I.random_kv_layer(d, 1, P, l, seed + 10 * b)
            ks.append(k[0].astype(np.float64))
            vs.append(v[0].astype(np.float64))
        out.append((ks, vs))
    return out


@pytest.fixture(scope="module")
def setup():
    w = I.Weights(D, seed=0, gain_jitter=0.1)
    a, eps, t, mask = I.train_batch(D, 2)
    caches = _caches(D, 2)
    res = T.train_step(w, caches, a, eps, t, mask, ki=False)
    return w, caches, a, eps, t, mask, res


def _param(w, key):
    return np.asarray(w.head()[key[1]] if key[0] == "head" else w.layer(1, key[0])[key[1]], np.float64)


def _set(w, key, val):
    if key[0] == "head":
        w.overrides[("head", key[1])] = val
    else:
        w.overrides[(1, key[0], key[1])] = val


def _richardson(f, h):
    """Directional derivative of f at 0: central differences at h and h/2 combined so that the h^2
    error terms cancel (error O(h^4), rounding ~ 1e-16 |f| / h)."""
    d1 = (f(h) - f(-h)) / (2 * h)
    d2 = (f(h / 2) - f(-h / 2)) / h
    return (4 * d2 - d1) / 3


def _fd(w, key, caches, a, eps, t, mask, h=1e-3):
    base = _param(w, key)
    rng = np.random.default_rng(sum(map(ord, str(key))))
    delta = rng.standard_normal(base.shape) * max(float(np.std(base)), 0.02)

    def f(s):
        _set(w, key, base + s * delta)
        return T.loss_only(w, caches, a, eps, t, mask)
    fd = _richardson(f, h)
    _set(w, key, base)
    return fd, delta


def test_forward_loss_matches_the_dm0_velocity(setup):
    w, caches, a, eps, t, mask, res = setup
    ref = T.loss_only(w, caches, a, eps, t, mask)
    assert abs(res["loss"] - ref) <= 1e-12 * ref


@pytest.mark.parametrize("key", [("head", k) for k in T.HEAD_PARAMS]
                         + [(l, k) for l in range(D.layers) for k in T.LAYER_PARAMS])
def test_gradient_matches_finite_differences(setup, key):
    w, caches, a, eps, t, mask, res = setup
    fd, delta = _fd(w, key, caches, a, eps, t, mask)
    an = float(np.sum(res["grads"][key] * delta))
    assert abs(fd - an) <= 1e-7 * abs(an) + 2e-12, (key, fd, an)


@pytest.mark.parametrize("layer", range(D.layers))
def test_cache_gradient_matches_finite_differences(setup, layer):
    w, caches, a, eps, t, mask, res = setup
    rng = np.random.default_rng(40 + layer)
    for which in (0, 1):                                   # K, then V
        b = 1
        base = caches[b][which][layer]
        delta = rng.standard_normal(base.shape)

        def f(s):
            c2 = [(list(ks), list(vs)) for ks, vs in caches]
            c2[b][which][layer] = base + s * delta
            return T.loss_only(w, c2, a, eps, t, mask)
        fd = _richardson(f, 1e-3)
        an = float(np.sum(res["kv_grads"][b][layer][which] * delta))
        assert abs(fd - an) <= 1e-7 * abs(an) + 2e-12, (layer, which, fd, an)


def test_knowledge_insulation_changes_only_the_cache_gradient(setup):
    w, caches, a, eps, t, mask, res = setup
    ki = T.train_step(w, caches, a, eps, t, mask, ki=True)
    assert ki["kv_grads"] is None and ki["loss"] == res["loss"]
    for k, g in res["grads"].items():
        assert np.array_equal(ki["grads"][k], g)


def test_interpolation_end_points():
    rng = np.random.default_rng(1)
    a, eps = rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    x1, u1 = T.interpolate(a, eps, 1.0)
    x0, u0 = T.interpolate(a, eps, 0.0)
    assert np.array_equal(x1, eps) and np.array_equal(x0, a)     # pure noise at t = 1, data at t = 0
    assert np.array_equal(u1, eps - a) and np.array_equal(u0, eps - a)
    xm, _ = T.interpolate(a, eps, 0.25)
    np.testing.assert_allclose(xm, 0.25 * eps + 0.75 * a, rtol=1e-15, atol=1e-15)


def test_constant_velocity_closed_form():
    # W_out = 0: v = b_out for every token, so L = sum_valid (b_out - u)^2 / N and dL/db_out =
    # 2 sum_valid (b_out - u) / N; nothing upstream of the output projection gets a gradient
    w = I.Weights(D, seed=0)
    w.overrides[("head", "W_out")] = np.zeros((D.action_dim, D.hidden_a))
    a, eps, t, mask = I.train_batch(D, 2, seed=4100)
    res = T.train_step(w, _caches(D, 2), a, eps, t, mask)
    c = np.asarray(w.head()["b_out"], np.float64)
    r = np.where(mask, c[None, None, :] - (eps.astype(np.float64) - a), 0.0)
    n = mask.sum()
    assert abs(res["loss"] - np.sum(r * r) / n) <= 1e-13 * res["loss"]
    np.testing.assert_allclose(res["grads"][("head", "b_out")], 2 * r.sum(axis=(0, 1)) / n, rtol=1e-12)
    for k, g in res["grads"].items():
        if k not in (("head", "b_out"), ("head", "W_out")):
            assert not np.any(g), k


def test_empty_mask_gives_zero_loss_and_gradients():
    w = I.Weights(D, seed=0)
    a, eps, t, mask = I.train_batch(D, 1)
    res = T.train_step(w, _caches(D, 1), a, eps, t, np.zeros_like(mask), ki=False)
    assert res["loss"] == 0.0
    assert all(not np.any(g) for g in res["grads"].values())
    assert all(not np.any(x) for pair in res["kv_grads"][0] for x in pair)


def test_loss_is_normalised_over_the_valid_entries_of_the_batch():
    # L_batch = sum_b N_b L_b / sum_b N_b (not the mean of per-sample means), and the same for grads
    w = I.Weights(D, seed=0)
    a, eps, t, mask = I.train_batch(D, 2, seed=4200)
    caches = _caches(D, 2)
    both = T.train_step(w, caches, a, eps, t, mask)
    parts = [T.train_step(w, caches[b:b + 1], a[b:b + 1], eps[b:b + 1], t[b:b + 1], mask[b:b + 1])
             for b in range(2)]
    n = [int(mask[b].sum()) for b in range(2)]
    assert n[0] != n[1]
    want = (n[0] * parts[0]["loss"] + n[1] * parts[1]["loss"]) / sum(n)
    assert abs(both["loss"] - want) <= 1e-13 * want
    for k in both["grads"]:
        np.testing.assert_allclose(both["grads"][k], (n[0] * parts[0]["grads"][k] + n[1] * parts[1]["grads"][k]) / sum(n),
                                   rtol=1e-10, atol=1e-16)


def test_masked_entries_do_not_reach_the_loss():
    # the velocity target of a masked-out entry can be anything: move u there (through eps only where
    # the mask is off, and a to keep x_t fixed) and nothing changes
    w = I.Weights(D, seed=0)
    a, eps, t, mask = I.train_batch(D, 1, seed=4300)
    caches = _caches(D, 1)
    base = T.train_step(w, caches, a, eps, t, mask)
    a2, eps2 = a.astype(np.float64).copy(), eps.astype(np.float64).copy()
    off = ~mask
    # keep x_t = t eps + (1 - t) a fixed while changing u = eps - a at the masked-out entries
    eps2[off] += (1.0 - t[0]) * 3.0
    a2[off] -= t[0] * 3.0
    moved = T.train_step(w, caches, a2, eps2, t, mask)
    assert abs(moved["loss"] - base["loss"]) <= 1e-13 * base["loss"]
    for k, g in base["grads"].items():
        np.testing.assert_allclose(moved["grads"][k], g, rtol=1e-9, atol=1e-15)
