"""The bf16 rounding points of the CUDA path, emulated on the CPU (test infrastructure only).

The kernels keep residual streams, sums of squares, accumulators and the Euler state in fp32 and
round to bf16 only where a value becomes a tensor-core operand or a stored bf16 tensor.  This
module re-runs the oracle's layer definitions with values rounded to bf16 at exactly those points
and in fp64 everywhere else, so its distance from the oracle is the part of the GPU's distance that
bf16 causes.  The GPU's own fp32 accumulation adds ~1e-7 relative on top, far below it.  The GPU
tests take their depth-dependent tolerances from this emulation
(tests/test_tolerance_emulation_cpu.py checks every such bar against it).

Rounding points, per layer of either branch:
  1. the pending RMSNorm's operand bf16(g * h), 1/rms applied after the projection;
  2. q and k after QK-norm and RoPE, and v after 1/rms (the cache, and the attention operands);
  3. the softmax weights exp(s - m) before the PV product (their row sum stays unrounded);
  4. the attention output (the O-projection operand); the single-observation Euler loop also
     rounds each key split's normalised partial output before combining the splits;
  5. the SwiGLU output (the down-projection operand).

It uses the oracle's element functions (rms_norm, rope, silu, time embedding, Euler times) and
nothing of the CUDA path.
"""
from __future__ import annotations

import numpy as np

from oracle import dm0_oracle as O
from synth.inputs import round_bf16

F = np.float64


def rb(x):
    """Round to the nearest bf16 value (ties to even), back in fp64."""
    return round_bf16(np.asarray(x, np.float32)).astype(F)


def _norm_operand(h, g, eps):
    """(bf16(g * h), 1/rms(h)) of a pending RMSNorm: the GEMM operand and the scale applied after it."""
    h = np.asarray(h, F)
    inv = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)
    return rb(np.asarray(g, F) * h), inv


def qkv(w, h, positions, d):
    """Q/K/V of one branch as the QKV epilogue writes them (bf16), from the bf16 norm operand."""
    T, D = h.shape[0], d.head_dim
    x, inv = _norm_operand(h, w["attn_norm"], d.rms_eps)
    q = (x @ np.asarray(w["Wq"], F).T * inv).reshape(T, d.n_q, D).transpose(1, 0, 2)
    k = (x @ np.asarray(w["Wk"], F).T * inv).reshape(T, d.n_kv, D).transpose(1, 0, 2)
    v = (x @ np.asarray(w["Wv"], F).T * inv).reshape(T, d.n_kv, D).transpose(1, 0, 2)
    q = rb(O.rope(O.rms_norm(q, w["q_norm"], d.rms_eps), positions, d.rope_theta))
    k = rb(O.rope(O.rms_norm(k, w["k_norm"], d.rms_eps), positions, d.rope_theta))
    return q, k, rb(v)


def attention(q, k, v, key_splits=1, prefix=None):
    """Every query row over all keys (the mask is expressed by which keys are passed), bf16 softmax
    weights in the PV product.  With key_splits > 1 (the single-launch Euler loop) the keys are cut into
    64-key blocks (the first `prefix` keys, then the rest as one more block, as the loop walks [prefix
    cache; suffix]), the blocks into key_splits contiguous ranges, and each range's normalised output is
    rounded to bf16 before the exact combine."""
    Hq, Tq, D = q.shape
    G = Hq // k.shape[0]
    Tk = k.shape[1]
    P = Tk if prefix is None else prefix
    starts = list(range(0, P, 64)) + ([P] if P < Tk else [])
    ends = starts[1:] + [Tk]
    nblk = len(starts)
    bps = -(-nblk // key_splits)
    bounds = [(starts[b0], ends[min(nblk, b0 + bps) - 1]) for b0 in range(0, nblk, bps)]
    out = np.empty((Hq, Tq, D), F)
    for h in range(Hq):
        j = h // G
        s = (q[h] @ k[j].T) / np.sqrt(F(D))
        if len(bounds) == 1:
            m = s.max(axis=-1, keepdims=True)
            e = np.exp(s - m)
            out[h] = (rb(e) @ v[j]) / e.sum(axis=-1, keepdims=True)
            continue
        parts, ms, ls = [], [], []
        for a, b in bounds:
            m = s[:, a:b].max(axis=-1, keepdims=True)
            e = np.exp(s[:, a:b] - m)
            lsum = e.sum(axis=-1, keepdims=True)
            parts.append(rb((rb(e) @ v[j][a:b]) / lsum))
            ms.append(m)
            ls.append(lsum)
        mx = np.max(np.concatenate(ms, axis=-1), axis=-1, keepdims=True)
        wts = [lsum * np.exp(m - mx) for m, lsum in zip(ms, ls)]
        den = sum(wts)
        out[h] = sum(wt * p for wt, p in zip(wts, parts)) / den
    return rb(out)


def finish(w, h, o, d, fp8=False):
    """O-projection + residual, then the MLP with its bf16 norm operand and bf16 SwiGLU output; with
    fp8 the VLM's E4M3 MLP instead, whose operands the GPU quantises from fp32 (the normalised residual
    and the SwiGLU output), with its code decisions in fp32 as the oracle's quantize_rows_f32 takes them."""
    T = h.shape[0]
    h = np.asarray(h, F) + o.transpose(1, 0, 2).reshape(T, d.n_q * d.head_dim) @ np.asarray(w["Wo"], F).T
    if fp8:
        return h + O.mlp_fp8(w, O.rms_norm(h, w["mlp_norm"], d.rms_eps), qrows=O.quantize_rows_f32)
    x, inv = _norm_operand(h, w["mlp_norm"], d.rms_eps)
    gate = x @ np.asarray(w["Wg"], F).T * inv
    up = x @ np.asarray(w["Wu"], F).T * inv
    return h + rb(O.silu(gate) * up) @ np.asarray(w["Wd"], F).T


def prefill(weights, prefix_emb, fp8=False):
    """The prefix pass of one sample as the GPU rounds it (fp8: with the E4M3 VLM MLP): ([k_l], [v_l], h)."""
    d = weights.d
    h = np.asarray(prefix_emb, F)
    P = h.shape[0]
    ks, vs = [], []
    for l in range(d.layers):
        w = weights.layer(0, l)
        q, k, v = qkv(w, h, np.arange(P), d)
        ks.append(k)
        vs.append(v)
        h = finish(w, h, attention(q, k, v), d, fp8)
    return ks, vs, h


def vlm_layer(w, h, d, fp8=False):
    """The VLM branch of one merged layer (prefix rows see the prefix only): (h', k, v)."""
    P = h.shape[0]
    q, k, v = qkv(w, h, np.arange(P), d)
    return finish(w, h, attention(q, k, v), d, fp8), k, v


def velocity(weights, ks, vs, x, t, key_splits=1):
    """The action expert's velocity over a cached prefix, as the GPU rounds it."""
    d = weights.d
    head = weights.head()
    h = O.action_input(head, x, t, d)
    P = ks[0].shape[1]
    S = h.shape[0]
    for l in range(d.layers):
        w = weights.layer(1, l)
        q, k, v = qkv(w, h, np.arange(P, P + S), d)
        k_all = np.concatenate([np.asarray(ks[l], F), k], axis=1)
        v_all = np.concatenate([np.asarray(vs[l], F), v], axis=1)
        h = finish(w, h, attention(q, k_all, v_all, key_splits, prefix=P), d)
    return O.action_output(head, h, d)


def denoise(weights, ks, vs, noise, steps, key_splits=1):
    """The Euler loop of one sample with the emulated velocity: (x_0, [v_k])."""
    x = np.asarray(noise, F)
    dt = -1.0 / steps
    vels = []
    for t in O.euler_times(steps):
        v = velocity(weights, ks, vs, x, t, key_splits)
        vels.append(v)
        x = x + dt * v
    return x, vels
