"""Plain fp64 CPU oracle of the DM0 dual-expert merged-attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module; only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg use it.  It shares no code with the CUDA path: the only common
dependency is the seeded input generator in synth/inputs.py.

Sources (page title and section):
  [DM0-arch]  DM0 architecture notes, dregs-remover.com/news/27019, section 1
              ("most important architecture conclusions"): each of the two
              Qwen3 experts makes its own Q/K/V in every layer, the two sets are
              concatenated along the sequence axis, run through one attention,
              split back, and each branch applies its own O-proj, residual and
              MLP; DM0-base shapes (28 layers, hidden 2048 / 1024, 16 heads,
              8 KV heads, head_dim 128, action dim 32, chunk 50).
  [DM05]      "DM0.5: High-Performance Embodied VLA and OpenDM Open Source
              Introduction", section 5.1 (prefix pass builds the VLM KV cache
              once), 5.2 (action_in_proj -> action expert -> action_out_proj ->
              velocity), 5.3 (flow matching: x_t = t*eps + (1-t)*a,
              u_t = eps - a, Euler integration from x_1 with diffusion_steps=10),
              6.2 (the suffix reads the prefix cache while processing the chunk).

Readings of points the pages leave open:
  R1 RMSNorm: x / sqrt(mean(x^2) + eps) * g, eps 1e-6 (Qwen3 default).
  R2 RoPE: rotate-half pairing (i, i + D/2), inv_freq_i = theta^(-2i/D),
     theta 1e6; prefix positions 0..P-1, suffix positions P..P+S-1.
  R3 QK-norm: RMSNorm over head_dim with per-branch gains, before RoPE.
  R4 GQA: query head h reads KV head floor(h / (n_q / n_kv)).
  R5 Block mask: prefix rows see prefix keys only; suffix rows see all P+S
     keys; no causal order inside either block; concatenation [prefix; suffix].
  R6 Time embedding tau(t) in R^{H_a}: half = H_a/2, w_i = 10000^(-i/half),
     tau = [sin(t w), cos(t w)], raw t (no scaling, no MLP), added to
     action_in_proj(x) + b_in and broadcast over the chunk.
  R7 action_in_proj and action_out_proj carry biases; a final RMSNorm (own
     gain) precedes action_out_proj.
  R8 Euler: t_k = 1 - k/K (k = 0..K-1), x <- x + dt * v(x, t_k), dt = -1/K;
     integration runs from noise (t=1) to data (t=0) because dx/dt = u = eps-a.
  R9 The KV cache holds K after QK-norm and RoPE, and V.
  R11 (the FP8 prefix MLP, a next step; [DM05] 6.3 names FP8 E4M3 for the gate/up/down GEMMs
     with scales but gives no scaling scheme): OCP E4M3 values (1-4-3, exponent bias 7, no
     infinities, largest finite 448), round to nearest with ties to even, saturating at +-448;
     per-token activation scales and per-output-channel weight scales, s = amax(|row|) / 448;
     products accumulated wide (fp64 here).

Precision: fp64 throughout.  Weights are the bf16-representable values from
synth/inputs.py, upcast.  No blocking, fusion or reordering beyond the
definitions: a matmul is a library primitive, softmax is written out.
"""
from __future__ import annotations

import numpy as np

F = np.float64


def rms_norm(x, g, eps):
    """R1 (Qwen3 RMSNorm) over the last axis."""
    x = np.asarray(x, F)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, F)


def rope(x, positions, theta):
    """R2: rotate-half RoPE. x [..., T, D], positions [T]."""
    x = np.asarray(x, F)
    D = x.shape[-1]
    half = D // 2
    inv_freq = np.asarray(theta, F) ** (-2.0 * np.arange(half, dtype=F) / D)
    ang = np.asarray(positions, F)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x):
    return x / (1.0 + np.exp(-x))


def attention(q, k, v, visible):
    """Softmax attention with GQA (R4). q [Hq,Tq,D], k/v [Hkv,Tk,D], visible [Tq,Tk] bool."""
    Hq, Tq, D = q.shape
    Hkv = k.shape[0]
    group = Hq // Hkv
    out = np.empty((Hq, Tq, D), F)
    for h in range(Hq):
        j = h // group
        s = (q[h] @ k[j].T) / np.sqrt(F(D))
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        out[h] = p @ v[j]
    return out


def project_qkv(w, h, positions, d):
    """Per-branch pre-norm, Q/K/V projections, QK-norm (R3) and RoPE (R2).

    h [T, H] -> q [Hq, T, D], k [Hkv, T, D], v [Hkv, T, D].  [DM0-arch]: each
    branch makes its own Q/K/V with the same head count and head_dim.
    """
    return qkv_from_normed(w, rms_norm(h, w["attn_norm"], d.rms_eps), positions, d)


def qkv_from_normed(w, r, positions, d):
    """The part of project_qkv after the pre-norm: r [T, H] (the normalised residual) -> q, k, v."""
    T = r.shape[0]
    D = d.head_dim
    q = (r @ np.asarray(w["Wq"], F).T).reshape(T, d.n_q, D).transpose(1, 0, 2)
    k = (r @ np.asarray(w["Wk"], F).T).reshape(T, d.n_kv, D).transpose(1, 0, 2)
    v = (r @ np.asarray(w["Wv"], F).T).reshape(T, d.n_kv, D).transpose(1, 0, 2)
    q = rope(rms_norm(q, w["q_norm"], d.rms_eps), positions, d.rope_theta)
    k = rope(rms_norm(k, w["k_norm"], d.rms_eps), positions, d.rope_theta)
    return q, k, v


def finish_layer(w, h, o, d, fp8=None):
    """Branch-own O-proj + residual, then pre-norm SwiGLU MLP + residual. o [Hq, T, D].

    fp8: None for the plain MLP; True for the E4M3 MLP of R11 (mlp_fp8); a row quantiser (as qrows of
    gemm_e4m3) for the E4M3 MLP with that quantiser."""
    T = h.shape[0]
    o_flat = o.transpose(1, 0, 2).reshape(T, d.n_q * d.head_dim)
    h = np.asarray(h, F) + o_flat @ np.asarray(w["Wo"], F).T
    r = rms_norm(h, w["mlp_norm"], d.rms_eps)
    if fp8 is not None:
        return h + mlp_fp8(w, r, qrows=None if fp8 is True else fp8)
    gate = r @ np.asarray(w["Wg"], F).T
    up = r @ np.asarray(w["Wu"], F).T
    return h + (silu(gate) * up) @ np.asarray(w["Wd"], F).T


def block_mask(P, S):
    """R5: [P+S, P+S] visibility of the concatenated [prefix; suffix] sequence."""
    vis = np.zeros((P + S, P + S), dtype=bool)
    vis[:P, :P] = True
    vis[P:, :] = True
    return vis


def merged_layer(wv, wa, h_prefix, h_suffix, d, vlm_fp8=None):
    """One dual-expert layer over the explicitly concatenated sequence ([DM0-arch]).

    h_prefix [P, Hv], h_suffix [S, Ha] (one sample).  Returns
    (h_prefix', h_suffix', k_prefix [Hkv,P,D], v_prefix [Hkv,P,D]).  vlm_fp8 selects the VLM
    branch's E4M3 MLP as finish_layer's fp8 does (the action branch stays plain).
    """
    P, S = h_prefix.shape[0], h_suffix.shape[0]
    qv, kv, vv = project_qkv(wv, h_prefix, np.arange(P), d)
    qa, ka, va = project_qkv(wa, h_suffix, np.arange(P, P + S), d)
    q = np.concatenate([qv, qa], axis=1)
    k = np.concatenate([kv, ka], axis=1)
    v = np.concatenate([vv, va], axis=1)
    o = attention(q, k, v, block_mask(P, S))
    return (finish_layer(wv, h_prefix, o[:, :P], d, vlm_fp8),
            finish_layer(wa, h_suffix, o[:, P:], d), kv, vv)


def prefill(weights, prefix_emb):
    """Prefix pass of one sample ([DM05] 5.1): the VLM alone over the prefix.

    Because prefix rows never see suffix keys (R5), this equals the prefix
    half of the merged forward.  Returns ([k_l], [v_l], h_final), k_l/v_l
    [Hkv, P, D] per layer (R9).
    """
    d = weights.d
    h = np.asarray(prefix_emb, F)
    P = h.shape[0]
    ks, vs = [], []
    vis = np.ones((P, P), dtype=bool)
    for l in range(d.layers):
        w = weights.layer(0, l)
        q, k, v = project_qkv(w, h, np.arange(P), d)
        ks.append(k)
        vs.append(v)
        h = finish_layer(w, h, attention(q, k, v, vis), d)
    return ks, vs, h


def time_embedding(t, H):
    """R6: sinusoidal embedding of the flow time t, size H."""
    half = H // 2
    omega = F(10000.0) ** (-np.arange(half, dtype=F) / half)
    return np.concatenate([np.sin(F(t) * omega), np.cos(F(t) * omega)])


def action_input(head, x, t, d):
    """[DM05] 5.2 action_in_proj plus the time embedding (R6, R7). x [S, A] -> [S, Ha]."""
    return (np.asarray(x, F) @ np.asarray(head["W_in"], F).T + np.asarray(head["b_in"], F)
            + time_embedding(t, d.hidden_a)[None, :])


def action_output(head, h, d):
    """[DM05] 5.2 final norm + action_out_proj -> velocity (R7). h [S, Ha] -> [S, A]."""
    r = rms_norm(h, head["final_norm"], d.rms_eps)
    return r @ np.asarray(head["W_out"], F).T + np.asarray(head["b_out"], F)


def suffix_layer(w, h, k_cache, v_cache, d):
    """Action-expert layer of the merged attention, suffix rows only ([DM0-arch], [DM05] 6.2).

    Suffix rows see every prefix key and every suffix key (R5), so this is
    the suffix half of merged_layer with the prefix K/V read from the cache.
    """
    P, S = k_cache.shape[1], h.shape[0]
    q, k, v = project_qkv(w, h, np.arange(P, P + S), d)
    k_all = np.concatenate([np.asarray(k_cache, F), k], axis=1)
    v_all = np.concatenate([np.asarray(v_cache, F), v], axis=1)
    o = attention(q, k_all, v_all, np.ones((S, P + S), dtype=bool))
    return finish_layer(w, h, o, d)


def velocity(weights, ks, vs, x, t):
    """v_theta(x_t, t | c) of one sample ([DM05] 5.2) over the cached prefix K/V."""
    d = weights.d
    head = weights.head()
    h = action_input(head, x, t, d)
    for l in range(d.layers):
        h = suffix_layer(weights.layer(1, l), h, ks[l], vs[l], d)
    return action_output(head, h, d)


def euler_times(steps):
    """R8: t_k = 1 - k/K, k = 0..K-1, each computed directly."""
    return [1.0 - k / steps for k in range(steps)]


def denoise(weights, ks, vs, noise, steps):
    """[DM05] 5.3 Euler sampler for one sample: x_1 = noise, x <- x + dt*v, dt = -1/K (R8).

    Returns (x_0 [S, A], [v_k] per step).
    """
    x = np.asarray(noise, F)
    dt = -1.0 / steps
    vels = []
    for t in euler_times(steps):
        v = velocity(weights, ks, vs, x, t)
        vels.append(v)
        x = x + dt * v
    return x, vels


def infer(weights, prefix_emb, noise, steps):
    """Observation -> action chunk for a batch: prefill once, then the Euler loop per sample.

    prefix_emb [B, P, Hv], noise [B, S, A].  Returns (chunks [B,S,A], caches, velocities).
    """
    chunks, caches, vels = [], [], []
    for b in range(prefix_emb.shape[0]):
        ks, vs, _ = prefill(weights, prefix_emb[b])
        x, v = denoise(weights, ks, vs, noise[b], steps)
        chunks.append(x)
        caches.append((ks, vs))
        vels.append(v)
    return np.stack(chunks), caches, vels


# ---------------------------------------------------------------- FP8 E4M3 prefix MLP (reading R11)

E4M3_MAX = 448.0


def e4m3(x):
    """R11: x rounded to the nearest FP8 E4M3 value (ties to even), saturating at +-448.

    Representable magnitudes are m 2^(e-3) for e in [-6, 8] and integer m in [8, 15] (normals), and
    m 2^-9 for m in [0, 7] (subnormals): the spacing at |x| is 2^(floor(log2|x|) - 3), clamped below
    to the subnormal spacing 2^-9 and above to that of the top binade, 2^5.
    """
    x = np.asarray(x, F)
    a = np.abs(x)
    e = np.clip(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6, 8)
    step = np.exp2(e - 3)
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)   # numpy rint: ties to even
    return np.copysign(q, x)


def quantize_rows(x, quant=e4m3):
    """R11: per-row scale s = amax(|row|) / 448 (1 for an all-zero row) and the codes quant(x / s)."""
    x = np.asarray(x, F)
    amax = np.max(np.abs(x), axis=-1, keepdims=True)
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return quant(x / s), s


def quantize_rows_f32(x):
    """R11 with the decision taken in fp32, the precision of the GPU quantiser: a code is an integer
    decided by floating point, so for code-level parity both sides decide it the same way.  The scale
    is fp32(amax) / 448 and the quotient x / scale an fp32 division (IEEE, correctly rounded in both
    numpy and the GPU), then rounded to E4M3 as in e4m3()."""
    x32 = np.asarray(x, np.float32)
    amax = np.max(np.abs(x32), axis=-1, keepdims=True)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    return e4m3((x32 / s).astype(F)), s.astype(F)


def gemm_e4m3(x, w, quant=e4m3, qrows=None):
    """x [T, K] @ w[N, K]^T with both operands quantised (per-token / per-output-channel scales, R11)
    and the products of the codes summed in fp64, then rescaled.  qrows(m) -> (codes, scales) replaces
    the row quantiser (default: quantize_rows with the element rounding `quant`)."""
    if qrows is None:
        def qrows(m):
            return quantize_rows(m, quant)
    xq, sx = qrows(x)
    wq, sw = qrows(w)
    return (xq @ wq.T) * sx * sw.T


def mlp_fp8(w, r, quant=e4m3, qrows=None):
    """[DM05] 6.3 with reading R11: the SwiGLU MLP of a VLM layer with its gate, up and down GEMMs in
    E4M3.  r [T, Hv] is the MLP's RMSNorm output; returns the MLP output (the residual add is the
    caller's)."""
    gate = gemm_e4m3(r, w["Wg"], quant, qrows)
    up = gemm_e4m3(r, w["Wu"], quant, qrows)
    return gemm_e4m3(silu(gate) * up, w["Wd"], quant, qrows)


def prefill_fp8(weights, prefix_emb, qrows=None):
    """The prefix pass (as prefill) with every VLM MLP in E4M3 (R11): the attention half of each layer
    is unchanged, the MLP is mlp_fp8 of the MLP's RMSNorm output (qrows as in gemm_e4m3).  Returns
    ([k_l], [v_l], h_final)."""
    d = weights.d
    h = np.asarray(prefix_emb, F)
    P = h.shape[0]
    ks, vs = [], []
    vis = np.ones((P, P), dtype=bool)
    for l in range(d.layers):
        w = weights.layer(0, l)
        q, k, v = project_qkv(w, h, np.arange(P), d)
        ks.append(k)
        vs.append(v)
        h = finish_layer(w, h, attention(q, k, v, vis), d, True if qrows is None else qrows)
    return ks, vs, h

