"""Plain fp64 CPU oracle of the DM0.5 time-modulated action expert (a next step after the DM0 path).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this module; only tests/,
__graft_entry__.smoke() and bench.py's CPU baseline leg use it.  It shares no code with the CUDA path.

Source: "DM0.5: High-Performance Embodied VLA and OpenDM Open Source Introduction", section 5.2: the
action expert turns the flow time step into a modulation signal with two layers, time_mlp_in and
time_mlp_out, and every layer carries a time modulator that tells the expert where on the noisy
trajectory it is; action_in_proj and action_out_proj surround the stack; section 5.3 for the Euler
sampler (unchanged from the DM0 oracle).

Reading R12 (the page names the modules but gives no formula; this is the plainest form that fits it,
the adaptive-RMSNorm modulation of diffusion transformers):
  c(t)    = W_to silu(W_ti tau(t) + b_ti) + b_to           tau from R6, both layers hidden_a -> hidden_a
  [g|b|a] = W_m silu(c) + b_m                             one modulator per pre-norm, hidden_a -> 3 hidden_a
  norm    = x / sqrt(mean(x^2) + eps) * (1 + g) + b       replaces the static gain of that RMSNorm
  h      += a * sublayer(norm)                            the third vector gates the residual add
  The final RMSNorm before action_out_proj is modulated by [g|b] only (W_mf: hidden_a -> 2 hidden_a).
  Time enters only through the modulators: tau(t) is no longer added to action_in_proj(x) + b_in.
  QK-norms keep their static gains; the VLM branch and the prefix cache are unchanged.
Everything else (RMSNorm eps, RoPE, QK-norm, GQA, mask, Euler grid) follows the DM0 oracle's R1-R9.

Precision: fp64 throughout; matrices are the bf16-representable values from synth/inputs.py.
"""
from __future__ import annotations

import numpy as np

from . import dm0_oracle as O

F = np.float64


def time_condition(tw, t, d):
    """R12: c(t) = time_mlp_out(silu(time_mlp_in(tau(t)))), a vector of hidden_a."""
    tau = O.time_embedding(t, d.hidden_a)
    z = np.asarray(tw["W_ti"], F) @ tau + np.asarray(tw["b_ti"], F)
    return np.asarray(tw["W_to"], F) @ O.silu(z) + np.asarray(tw["b_to"], F)


def modulation(W, b, c, parts):
    """R12: W silu(c) + b split into `parts` consecutive vectors of hidden_a (scale, shift[, gate])."""
    m = np.asarray(W, F) @ O.silu(np.asarray(c, F)) + np.asarray(b, F)
    return np.split(m, parts)


def ada_rms(x, scale, shift, eps):
    """R12 modulated RMSNorm over the last axis: x / rms(x) * (1 + scale) + shift."""
    x = np.asarray(x, F)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * (1.0 + scale) + shift


def suffix_layer(w, m, c, h, k_cache, v_cache, d):
    """One time-modulated action layer over the cached prefix K/V (suffix rows see all P+S keys, R5)."""
    P, S = k_cache.shape[1], h.shape[0]
    h = np.asarray(h, F)
    g_a, b_a, a_a = modulation(m["W_ma"], m["b_ma"], c, 3)
    q, k, v = O.qkv_from_normed(w, ada_rms(h, g_a, b_a, d.rms_eps), np.arange(P, P + S), d)
    k_all = np.concatenate([np.asarray(k_cache, F), k], axis=1)
    v_all = np.concatenate([np.asarray(v_cache, F), v], axis=1)
    o = O.attention(q, k_all, v_all, np.ones((S, P + S), dtype=bool))
    o_flat = o.transpose(1, 0, 2).reshape(S, d.n_q * d.head_dim)
    h = h + a_a * (o_flat @ np.asarray(w["Wo"], F).T)
    g_m, b_m, a_m = modulation(m["W_mm"], m["b_mm"], c, 3)
    r = ada_rms(h, g_m, b_m, d.rms_eps)
    mlp = (O.silu(r @ np.asarray(w["Wg"], F).T) * (r @ np.asarray(w["Wu"], F).T)) @ np.asarray(w["Wd"], F).T
    return h + a_m * mlp


def velocity(weights, ks, vs, x, t):
    """v_theta(x_t, t | c) of one sample for the time-modulated expert (R12)."""
    d = weights.d
    head, tw = weights.head(), weights.time()
    c = time_condition(tw, t, d)
    h = np.asarray(x, F) @ np.asarray(head["W_in"], F).T + np.asarray(head["b_in"], F)
    for l in range(d.layers):
        h = suffix_layer(weights.layer(1, l), weights.mod(l), c, h, ks[l], vs[l], d)
    g_f, b_f = modulation(tw["W_mf"], tw["b_mf"], c, 2)
    return ada_rms(h, g_f, b_f, d.rms_eps) @ np.asarray(head["W_out"], F).T + np.asarray(head["b_out"], F)


def denoise(weights, ks, vs, noise, steps):
    """Euler sampler of the DM0 oracle (R8) driven by the time-modulated velocity.

    Returns (x_0 [S, A], [v_k] per step)."""
    x = np.asarray(noise, F)
    dt = -1.0 / steps
    vels = []
    for t in O.euler_times(steps):
        v = velocity(weights, ks, vs, x, t)
        vels.append(v)
        x = x + dt * v
    return x, vels
