"""The GPU decomposition of the time-modulated expert (dm0_denoise with time_mod = 1), emulated in numpy
against the fp64 oracle (oracle/dm05_oracle.py, reading R12).

The GPU never forms the modulated norm x / rms(x) (1 + scale) + shift itself: the GEMM operand stays
bf16((1 + scale) h) with 1/rms applied to the product, the shift enters as the feature bias
W bf16(shift) (computed once per Euler loop for every step), the gate scales the sublayer's output
before the residual add, and the final norm's shift goes through W_out.  The time MLP and the
modulators run on bf16 operands.  This checks the algebra of that rewrite and that its rounding stays
well inside the GPU tests' 2e-2 bar on the velocity.
"""
import numpy as np
import pytest

from oracle import dm0_oracle as O
from oracle import dm05_oracle as M
from synth import inputs as I

F = np.float64


def bf(x):
    """Round to the nearest bf16 value (the GPU's operand rounding)."""
    return I.round_bf16(np.asarray(x, np.float32)).astype(F)


def silu(x):
    return x / (1.0 + np.exp(-x))


def tables(w, t, d):
    """The per-step table the GPU builds: every norm's [1 + scale | shift | gate] and the final one."""
    tw = w.time()
    z = bf(O.time_embedding(t, d.hidden_a)) @ np.asarray(tw["W_ti"], F).T + tw["b_ti"]
    c = bf(silu(z)) @ np.asarray(tw["W_to"], F).T + tw["b_to"]
    sc = bf(silu(c))
    rows = []
    for l in range(d.layers):
        m = w.mod(l)
        rows.append((sc @ np.asarray(m["W_ma"], F).T + m["b_ma"], sc @ np.asarray(m["W_mm"], F).T + m["b_mm"]))
    fin = sc @ np.asarray(tw["W_mf"], F).T + tw["b_mf"]
    return rows, fin


def velocity_gpu_form(w, ks, vs, x, t, d):
    H = d.hidden_a
    rows, fin = tables(w, t, d)
    head = w.head()
    h = np.asarray(x, F) @ np.asarray(head["W_in"], F).T + head["b_in"]      # no time embedding
    P, S = ks[0].shape[1], h.shape[0]
    for l in range(d.layers):
        lw = w.layer(1, l)
        (ma, mm) = rows[l]
        inv = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + d.rms_eps)
        wqkv = np.concatenate([np.asarray(lw[k], F) for k in ("Wq", "Wk", "Wv")])
        raw = (bf((1.0 + ma[:H]) * h) @ wqkv.T) * inv + bf(ma[H:2 * H]) @ wqkv.T
        qd, kd = d.n_q * d.head_dim, d.n_kv * d.head_dim
        q = raw[:, :qd].reshape(S, d.n_q, d.head_dim).transpose(1, 0, 2)
        k = raw[:, qd:qd + kd].reshape(S, d.n_kv, d.head_dim).transpose(1, 0, 2)
        v = raw[:, qd + kd:].reshape(S, d.n_kv, d.head_dim).transpose(1, 0, 2)
        pos = np.arange(P, P + S)
        q = O.rope(O.rms_norm(q, lw["q_norm"], d.rms_eps), pos, d.rope_theta)
        k = O.rope(O.rms_norm(k, lw["k_norm"], d.rms_eps), pos, d.rope_theta)
        o = O.attention(q, np.concatenate([ks[l], k], axis=1), np.concatenate([vs[l], v], axis=1),
                        np.ones((S, P + S), dtype=bool))
        of = bf(o.transpose(1, 0, 2).reshape(S, qd))
        h = h + ma[2 * H:] * (of @ np.asarray(lw["Wo"], F).T)
        inv = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + d.rms_eps)
        wg, wu = np.asarray(lw["Wg"], F), np.asarray(lw["Wu"], F)
        op, sh = bf((1.0 + mm[:H]) * h), bf(mm[H:2 * H])
        g = (op @ wg.T) * inv + sh @ wg.T
        u = (op @ wu.T) * inv + sh @ wu.T
        h = h + mm[2 * H:] * (bf(silu(g) * u) @ np.asarray(lw["Wd"], F).T)
    inv = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + d.rms_eps)
    wo = np.asarray(head["W_out"], F)
    return ((1.0 + fin[:H]) * h) @ wo.T * inv + fin[H:] @ wo.T + head["b_out"]


@pytest.mark.parametrize("d,P", [(I.TINY, 16), (I.DM0_BASE.replace(layers=1), 64)])
@pytest.mark.parametrize("t", [1.0, 0.35])
def test_gpu_form_matches_the_modulated_oracle(d, P, t):
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    ks, vs = [], []
    for l in range(d.layers):
        k, v = I.random_kv_layer(d, 1, P, l)
        ks.append(k[0].astype(F))
        vs.append(v[0].astype(F))
    x = I.noise(d, 1)[0].astype(F)
    ref = M.velocity(w, ks, vs, x, t)
    got = velocity_gpu_form(w, ks, vs, x, t, d)
    err = np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref ** 2))
    print(f"max|d|/RMS = {err:.2e}")
    assert err <= 2e-2 / 4
