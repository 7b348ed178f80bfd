"""Plain fp64 CPU oracle of one flow-matching training step of the DM0 action expert (a next step).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this module; only tests/,
__graft_entry__.smoke() and bench.py's CPU baseline leg use it.  It shares no code with the CUDA path.

Sources (page title and section):
  "DM0.5: High-Performance Embodied VLA and OpenDM Open Source Introduction", section 5.3: the
  training input is the interpolation x_t = t eps + (1 - t) a between a real action chunk a and noise
  eps, the target is u_t = eps - a, the loss is the mean squared error between v_theta(x_t, t | c) and
  u_t, restricted by an action mask to the valid action dimensions and valid chunk positions.
  DM0 architecture notes (dregs-remover.com/news/27019), section 1: the paper's knowledge insulation
  keeps the action expert's gradient out of the VLM, while the public code shows no explicit stop
  gradient on the prefix K/V.

Reading R13 (points the pages leave open):
  - the loss of a batch is the sum of (v - u)^2 over all valid entries of all samples divided by the
    number of valid entries (0 when there are none);
  - t and eps are inputs (the pages give no distribution for t);
  - the step returns the loss and the gradient of every action-expert parameter (each layer's
    attn_norm, Wq, Wk, Wv, q_norm, k_norm, Wo, mlp_norm, Wg, Wu, Wd) and of the head (W_in, b_in,
    final_norm, W_out, b_out); the prefix K/V cache is a constant under knowledge insulation (the
    default); with ki=False the gradients with respect to each layer's cached K and V are returned
    as well, the point where the public code's graph would continue into the VLM (out of scope);
  - no optimiser update (the pages name none).
The forward is the DM0 oracle's velocity (readings R1-R9); the backward is the chain rule written
out by hand for each operation and is pinned by finite differences.

Precision: fp64 throughout.
"""
from __future__ import annotations

import numpy as np

from . import dm0_oracle as O

F = np.float64
LAYER_PARAMS = ("attn_norm", "Wq", "Wk", "Wv", "q_norm", "k_norm", "Wo", "mlp_norm", "Wg", "Wu", "Wd")
HEAD_PARAMS = ("W_in", "b_in", "final_norm", "W_out", "b_out")


def interpolate(a, eps, t):
    """[DM05] 5.3: the training input x_t and the velocity target u_t of one sample."""
    a, eps = np.asarray(a, F), np.asarray(eps, F)
    return t * eps + (1.0 - t) * a, eps - a


# ---------------------------------------------------------------- operations with their adjoints

def _rms_fwd(x, g, eps):
    """R1 RMSNorm, keeping the normalised input n = x rho and rho = (mean(x^2) + eps)^(-1/2)."""
    x = np.asarray(x, F)
    rho = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    n = x * rho
    return n * np.asarray(g, F), (n, rho)


def _rms_bwd(dy, g, saved):
    """y = g n, n = x rho: dn = g dy; dx = rho (dn - n mean(dn n)); dg = sum over rows of dy n."""
    n, rho = saved
    dn = dy * np.asarray(g, F)
    dx = rho * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    dg = np.sum((dy * n).reshape(-1, n.shape[-1]), axis=0)
    return dx, dg


def _rope_tables(positions, D, theta):
    half = D // 2
    inv_freq = F(theta) ** (-2.0 * np.arange(half, dtype=F) / D)
    ang = np.asarray(positions, F)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def _rope_fwd(x, c, s):
    """R2 rotate-half RoPE: each pair (i, i + D/2) is rotated by its angle."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _rope_bwd(dy, c, s):
    """The transpose of a rotation is the rotation by the opposite angle."""
    half = dy.shape[-1] // 2
    d1, d2 = dy[..., :half], dy[..., half:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


# ---------------------------------------------------------------- one action layer

def layer_forward(w, h, k_cache, v_cache, d):
    """Action layer over the cached prefix K/V (as the DM0 oracle's suffix_layer), keeping what the
    backward needs."""
    P, S = k_cache.shape[1], h.shape[0]
    Hq, Hkv, D = d.n_q, d.n_kv, d.head_dim
    W = {k: np.asarray(w[k], F) for k in ("Wq", "Wk", "Wv", "Wo", "Wg", "Wu", "Wd")}
    h = np.asarray(h, F)
    r1, s1 = _rms_fwd(h, w["attn_norm"], d.rms_eps)
    q3 = (r1 @ W["Wq"].T).reshape(S, Hq, D).transpose(1, 0, 2)
    k3 = (r1 @ W["Wk"].T).reshape(S, Hkv, D).transpose(1, 0, 2)
    v3 = (r1 @ W["Wv"].T).reshape(S, Hkv, D).transpose(1, 0, 2)
    qn, sq = _rms_fwd(q3, w["q_norm"], d.rms_eps)
    kn, sk = _rms_fwd(k3, w["k_norm"], d.rms_eps)
    cos, sin = _rope_tables(np.arange(P, P + S), D, d.rope_theta)
    qr, kr = _rope_fwd(qn, cos, sin), _rope_fwd(kn, cos, sin)
    K = np.concatenate([np.asarray(k_cache, F), kr], axis=1)
    V = np.concatenate([np.asarray(v_cache, F), v3], axis=1)
    group, scale = Hq // Hkv, 1.0 / np.sqrt(F(D))
    p = np.empty((Hq, S, P + S))
    o = np.empty((Hq, S, D))
    for hh in range(Hq):
        j = hh // group
        sc = (qr[hh] @ K[j].T) * scale
        e = np.exp(sc - sc.max(axis=-1, keepdims=True))
        p[hh] = e / e.sum(axis=-1, keepdims=True)
        o[hh] = p[hh] @ V[j]
    of = o.transpose(1, 0, 2).reshape(S, Hq * D)
    h1 = h + of @ W["Wo"].T
    r2, s2 = _rms_fwd(h1, w["mlp_norm"], d.rms_eps)
    gate, up = r2 @ W["Wg"].T, r2 @ W["Wu"].T
    sg = gate * _sigmoid(gate)
    act = sg * up
    h2 = h1 + act @ W["Wd"].T
    saved = dict(W=W, r1=r1, s1=s1, sq=sq, sk=sk, cos=cos, sin=sin, qr=qr, K=K, V=V, p=p, of=of,
                 r2=r2, s2=s2, gate=gate, up=up, sg=sg, act=act, P=P, S=S)
    return h2, saved


def layer_backward(w, c, dh2, d):
    """Adjoint of layer_forward: dh2 [S, H] -> (dh0, {param: grad}, dK_cache, dV_cache)."""
    W, P, S = c["W"], c["P"], c["S"]
    Hq, Hkv, D = d.n_q, d.n_kv, d.head_dim
    g = {}
    # MLP: h2 = h1 + act Wd^T, act = silu(gate) * up
    g["Wd"] = dh2.T @ c["act"]
    dact = dh2 @ W["Wd"]
    sig = _sigmoid(c["gate"])
    dgate = dact * c["up"] * sig * (1.0 + c["gate"] * (1.0 - sig))
    dup = dact * c["sg"]
    g["Wg"], g["Wu"] = dgate.T @ c["r2"], dup.T @ c["r2"]
    dr2 = dgate @ W["Wg"] + dup @ W["Wu"]
    dx, g["mlp_norm"] = _rms_bwd(dr2, w["mlp_norm"], c["s2"])
    dh1 = dh2 + dx
    # attention output projection: h1 = h0 + of Wo^T
    g["Wo"] = dh1.T @ c["of"]
    do = (dh1 @ W["Wo"]).reshape(S, Hq, D).transpose(1, 0, 2)
    # softmax attention per query head over its KV head
    group, scale = Hq // Hkv, 1.0 / np.sqrt(F(D))
    dK, dV = np.zeros_like(c["K"]), np.zeros_like(c["V"])
    dqr = np.empty_like(c["qr"])
    for hh in range(Hq):
        j = hh // group
        p = c["p"][hh]
        dp = do[hh] @ c["V"][j].T
        dV[j] += p.T @ do[hh]
        ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True)) * scale
        dqr[hh] = ds @ c["K"][j]
        dK[j] += ds.T @ c["qr"][hh]
    # RoPE and QK-norm of the suffix's own q and k; v went straight into V
    dq3, g["q_norm"] = _rms_bwd(_rope_bwd(dqr, c["cos"], c["sin"]), w["q_norm"], c["sq"])
    dk3, g["k_norm"] = _rms_bwd(_rope_bwd(dK[:, P:], c["cos"], c["sin"]), w["k_norm"], c["sk"])
    dqf = dq3.transpose(1, 0, 2).reshape(S, Hq * D)
    dkf = dk3.transpose(1, 0, 2).reshape(S, Hkv * D)
    dvf = dV[:, P:].transpose(1, 0, 2).reshape(S, Hkv * D)
    g["Wq"], g["Wk"], g["Wv"] = dqf.T @ c["r1"], dkf.T @ c["r1"], dvf.T @ c["r1"]
    dr1 = dqf @ W["Wq"] + dkf @ W["Wk"] + dvf @ W["Wv"]
    dx, g["attn_norm"] = _rms_bwd(dr1, w["attn_norm"], c["s1"])
    return dh1 + dx, g, dK[:, :P], dV[:, :P]


# ---------------------------------------------------------------- the step

def train_step(weights, caches, a, eps, t, mask, ki=True):
    """R13: loss and gradients of one flow-matching step over a batch.

    caches: per sample (ks, vs), ks[l] / vs[l] [Hkv, P, D]; a, eps [B, S, A]; t [B]; mask [B, S, A]
    bool.  Returns {"loss": L, "grads": {(l, name) | ("head", name): array}, "kv_grads": None or per
    sample [(dK_l, dV_l) per layer]}.
    """
    d = weights.d
    head = {k: np.asarray(v, F) for k, v in weights.head().items()}
    mask = np.asarray(mask, bool)
    n_valid = max(int(mask.sum()), 1)
    grads = {("head", k): np.zeros_like(head[k]) for k in HEAD_PARAMS}
    for l in range(d.layers):
        for k, v in weights.layer(1, l).items():
            grads[(l, k)] = np.zeros(np.shape(v), F)
    kv_grads = None if ki else []
    loss = 0.0
    for b in range(np.shape(a)[0]):
        ks, vs = caches[b]
        x_t, u = interpolate(a[b], eps[b], t[b])
        h = x_t @ head["W_in"].T + head["b_in"] + O.time_embedding(t[b], d.hidden_a)[None, :]
        saved = []
        for l in range(d.layers):
            h, c = layer_forward(weights.layer(1, l), h, ks[l], vs[l], d)
            saved.append(c)
        rf, sf = _rms_fwd(h, head["final_norm"], d.rms_eps)
        v = rf @ head["W_out"].T + head["b_out"]
        diff = np.where(mask[b], v - u, 0.0)
        loss += float(np.sum(diff * diff))
        dv = 2.0 * diff / n_valid
        grads[("head", "W_out")] += dv.T @ rf
        grads[("head", "b_out")] += dv.sum(axis=0)
        dh, dg = _rms_bwd(dv @ head["W_out"], head["final_norm"], sf)
        grads[("head", "final_norm")] += dg
        per_layer = [None] * d.layers
        for l in reversed(range(d.layers)):
            dh, gl, dkc, dvc = layer_backward(weights.layer(1, l), saved[l], dh, d)
            for k, gv in gl.items():
                grads[(l, k)] += gv
            per_layer[l] = (dkc, dvc)
        grads[("head", "W_in")] += dh.T @ x_t
        grads[("head", "b_in")] += dh.sum(axis=0)
        if kv_grads is not None:
            kv_grads.append(per_layer)
    return {"loss": loss / n_valid, "grads": grads, "kv_grads": kv_grads}


def loss_only(weights, caches, a, eps, t, mask):
    """The R13 loss through the DM0 oracle's own forward (velocity), without gradients."""
    mask = np.asarray(mask, bool)
    total = 0.0
    for b in range(np.shape(a)[0]):
        ks, vs = caches[b]
        x_t, u = interpolate(a[b], eps[b], t[b])
        v = O.velocity(weights, ks, vs, x_t, t[b])
        total += float(np.sum(np.where(mask[b], v - u, 0.0) ** 2))
    return total / max(int(mask.sum()), 1)
