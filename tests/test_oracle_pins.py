"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties the oracle to a library routine, a closed form, an invariant
the method guarantees, or a brute-force construction that shares none of the
oracle's structure.  Together they are chosen so that a plausible slip in the
oracle (a dropped QK-norm, interleaved instead of rotate-half RoPE, the wrong
GQA grouping, a leaky block mask, the wrong suffix positions, an Euler sign
flip, a missing final norm, sin/cos swapped) fails at least one of them.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

from oracle import dm0_oracle as O
from synth import inputs as I

@pytest.fixture(autouse=True)
def _fp64_default():
    """Library references in this module run in fp64; restore the default afterwards so that
    tests collected in the same session keep torch's fp32 default."""
    old = torch.get_default_dtype()
    torch.set_default_dtype(torch.float64)
    yield
    torch.set_default_dtype(old)


def _rms(x):
    return float(np.sqrt(np.mean(np.square(x))))


# ---------------------------------------------------------------- library routines

def test_rms_norm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 96))
    g = 1 + 0.1 * rng.standard_normal(96)
    ref = Fnn.rms_norm(torch.tensor(x), (96,), torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (8, 2)])
def test_attention_matches_sdpa_with_mask(hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    Tq, Tk, D = 9, 13, 16
    q = rng.standard_normal((hq, Tq, D))
    k = rng.standard_normal((hkv, Tk, D))
    v = rng.standard_normal((hkv, Tk, D))
    vis = rng.random((Tq, Tk)) < 0.6
    vis[:, 0] = True
    # library path: expand KV heads consecutively (query head h -> kv head h // (hq/hkv))
    rep = hq // hkv
    kt = torch.tensor(k).repeat_interleave(rep, dim=0)
    vt = torch.tensor(v).repeat_interleave(rep, dim=0)
    ref = Fnn.scaled_dot_product_attention(torch.tensor(q), kt, vt, attn_mask=torch.tensor(vis)).numpy()
    np.testing.assert_allclose(O.attention(q, k, v, vis), ref, rtol=1e-10, atol=1e-12)


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 4, 8))
    k = rng.standard_normal((1, 5, 8))
    v = rng.standard_normal((1, 5, 8))
    vis = np.zeros((4, 5), dtype=bool)
    vis[:, 3] = True
    out = O.attention(q, k, v, vis)
    np.testing.assert_array_equal(out, np.broadcast_to(v[0, 3], out.shape))


# ---------------------------------------------------------------- closed forms

def test_rope_closed_forms():
    D, theta = 32, 1e6
    x = np.zeros((1, D))
    x[0, 0] = 1.0
    # position 0 is the identity
    np.testing.assert_array_equal(O.rope(x, [0], theta), x)
    # frequency index 0 rotates the pair (0, D/2) by exactly the position angle
    p = 3.0
    y = O.rope(x, [p], theta)[0]
    assert abs(y[0] - np.cos(p)) < 1e-15 and abs(y[D // 2] - np.sin(p)) < 1e-15
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2
    # the last pair (D/2-1, D-1) turns at theta^(-(D-2)/D) per position
    x2 = np.zeros((1, D))
    x2[0, D - 1] = 1.0
    y2 = O.rope(x2, [1.0], theta)[0]
    a = theta ** (-(D - 2) / D)
    assert abs(y2[D - 1] - np.cos(a)) < 1e-15 and abs(y2[D // 2 - 1] + np.sin(a)) < 1e-15


def test_rope_relative_position_invariant():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 64))
    k = rng.standard_normal((1, 64))
    dots = [float((O.rope(q, [5 + s], 1e6) @ O.rope(k, [s], 1e6).T)[0, 0]) for s in (0, 7, 100)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


def test_time_embedding_closed_form():
    H = 128
    tau0 = O.time_embedding(0.0, H)
    np.testing.assert_array_equal(tau0, np.concatenate([np.zeros(H // 2), np.ones(H // 2)]))
    t = 0.7
    tau = O.time_embedding(t, H)
    assert abs(tau[0] - np.sin(t)) < 1e-15 and abs(tau[H // 2] - np.cos(t)) < 1e-15
    # the last frequency is 10000^(-(half-1)/half)
    w_last = 10000.0 ** (-(H // 2 - 1) / (H // 2))
    assert abs(tau[H // 2 - 1] - np.sin(t * w_last)) < 1e-15


def test_euler_time_grid():
    assert O.euler_times(4) == [1.0, 0.75, 0.5, 0.25]


# ---------------------------------------------------------------- transformers Qwen3 as a library pin

def _qwen3(d, branch, weights, layers=None, final_gain=None):
    from transformers import Qwen3Config, Qwen3Model
    cfg = Qwen3Config(vocab_size=8, hidden_size=d.hidden(branch), intermediate_size=d.inter(branch),
                      num_hidden_layers=layers or d.layers, num_attention_heads=d.n_q,
                      num_key_value_heads=d.n_kv, head_dim=d.head_dim, rms_norm_eps=d.rms_eps,
                      rope_theta=d.rope_theta, max_position_embeddings=4096, attention_bias=False,
                      attn_implementation="eager")
    cfg.rope_parameters = {"rope_type": "default", "rope_theta": d.rope_theta}
    m = Qwen3Model(cfg).to(torch.float64).eval()
    with torch.no_grad():
        for l, layer in enumerate(m.layers):
            w = weights.layer(branch, l)
            t = lambda a: torch.tensor(np.asarray(a, np.float64))
            layer.input_layernorm.weight.copy_(t(w["attn_norm"]))
            layer.self_attn.q_proj.weight.copy_(t(w["Wq"]))
            layer.self_attn.k_proj.weight.copy_(t(w["Wk"]))
            layer.self_attn.v_proj.weight.copy_(t(w["Wv"]))
            layer.self_attn.q_norm.weight.copy_(t(w["q_norm"]))
            layer.self_attn.k_norm.weight.copy_(t(w["k_norm"]))
            layer.self_attn.o_proj.weight.copy_(t(w["Wo"]))
            layer.post_attention_layernorm.weight.copy_(t(w["mlp_norm"]))
            layer.mlp.gate_proj.weight.copy_(t(w["Wg"]))
            layer.mlp.up_proj.weight.copy_(t(w["Wu"]))
            layer.mlp.down_proj.weight.copy_(t(w["Wd"]))
        m.norm.weight.copy_(torch.tensor(np.asarray(final_gain, np.float64)) if final_gain is not None
                            else torch.ones(d.hidden(branch)))
    return m


@pytest.fixture(scope="module")
def tiny_weights():
    return I.Weights(I.TINY, seed=0, gain_jitter=0.1)


def test_prefill_matches_transformers_qwen3(tiny_weights):
    d, P = I.TINY, 64
    emb = I.prefix_embeddings(d, 1, P)[0]
    ks, vs, h = O.prefill(tiny_weights, emb)
    m = _qwen3(d, 0, tiny_weights)
    from transformers import DynamicCache
    cache = DynamicCache(config=m.config)
    full = torch.zeros(1, 1, P, P)   # bidirectional prefix
    with torch.no_grad():
        out = m(inputs_embeds=torch.tensor(emb[None].astype(np.float64)),
                attention_mask={"full_attention": full}, past_key_values=cache, use_cache=True)
    ref_h = out.last_hidden_state[0].numpy()
    # the library applies its final norm (gain 1): compare against the normed oracle state
    got_h = O.rms_norm(h, np.ones(d.hidden_v), d.rms_eps)
    tol = 2e-5  # transformers builds cos/sin and softmax in fp32
    assert np.max(np.abs(got_h - ref_h)) <= tol * _rms(ref_h)
    for l in range(d.layers):
        kr = cache.layers[l].keys[0].numpy()
        vr = cache.layers[l].values[0].numpy()
        assert np.max(np.abs(ks[l] - kr)) <= tol * _rms(kr)
        assert np.max(np.abs(vs[l] - vr)) <= tol * _rms(vr)


def test_velocity_matches_transformers_qwen3_with_prefix_cache(tiny_weights):
    d, P = I.TINY, 64
    emb = I.prefix_embeddings(d, 1, P)[0]
    x = I.noise(d, 1)[0]
    ks, vs, _ = O.prefill(tiny_weights, emb)
    t = 0.75
    v_or = O.velocity(tiny_weights, ks, vs, x, t)
    head = tiny_weights.head()
    m = _qwen3(d, 1, tiny_weights, final_gain=head["final_norm"])
    from transformers import DynamicCache
    cache = DynamicCache(config=m.config)
    for l in range(d.layers):
        cache.update(torch.tensor(ks[l][None]), torch.tensor(vs[l][None]), l)
    S = d.chunk
    e = O.action_input(head, x, t, d)
    with torch.no_grad():
        out = m(inputs_embeds=torch.tensor(e[None]), attention_mask={"full_attention": torch.zeros(1, 1, S, P + S)},
                position_ids=torch.arange(P, P + S)[None], past_key_values=cache, use_cache=True)
    v_ref = out.last_hidden_state[0].numpy() @ head["W_out"].astype(np.float64).T + head["b_out"]
    assert np.max(np.abs(v_or - v_ref)) <= 2e-5 * _rms(v_ref)


# ---------------------------------------------------------------- brute force: merged sequence, no cache

def _bf_branch_qkv(layer, rot, h, pos):
    """q/k/v of one branch from transformers' Qwen3 layer modules (independent of the oracle)."""
    from transformers.models.qwen3.modeling_qwen3 import apply_rotary_pos_emb
    att = layer.self_attn
    T = h.shape[0]
    r = layer.input_layernorm(h[None])
    q = att.q_norm(att.q_proj(r).view(1, T, -1, att.head_dim)).transpose(1, 2)
    k = att.k_norm(att.k_proj(r).view(1, T, -1, att.head_dim)).transpose(1, 2)
    v = att.v_proj(r).view(1, T, -1, att.head_dim).transpose(1, 2)
    cos, sin = rot(h[None], torch.tensor(pos)[None])
    q, k = apply_rotary_pos_emb(q, k, cos, sin)
    return q, k, v


def _bf_branch_rest(layer, h, o):
    T = h.shape[0]
    h = h + layer.self_attn.o_proj(o.transpose(1, 2).reshape(1, T, -1))[0]
    return h + layer.mlp(layer.post_attention_layernorm(h[None]))[0]


def _brute_force_chunk(d, weights, emb, x, steps):
    """Every Euler step re-runs BOTH experts jointly over the explicit [prefix; suffix]
    sequence with one dense-mask SDPA per layer; no KV cache is kept."""
    mv, ma = _qwen3(d, 0, weights), _qwen3(d, 1, weights)
    head = weights.head()
    P, S = emb.shape[0], x.shape[0]
    mask = torch.zeros(P + S, P + S, dtype=torch.bool)
    mask[:P, :P] = True
    mask[P:, :] = True
    group = d.n_q // d.n_kv
    x = torch.tensor(x.astype(np.float64))
    vels = []
    for kstep in range(steps):
        t = 1.0 - kstep / steps
        half = d.hidden_a // 2
        w = 10000.0 ** (-torch.arange(half) / half)
        tau = torch.cat([torch.sin(t * w), torch.cos(t * w)])
        hv = torch.tensor(emb.astype(np.float64))
        ha = x @ torch.tensor(head["W_in"].astype(np.float64)).T + torch.tensor(head["b_in"].astype(np.float64)) + tau
        with torch.no_grad():
            for l in range(d.layers):
                qv, kv, vv = _bf_branch_qkv(mv.layers[l], mv.rotary_emb, hv, np.arange(P))
                qa, ka, va = _bf_branch_qkv(ma.layers[l], ma.rotary_emb, ha, np.arange(P, P + S))
                q = torch.cat([qv, qa], 2)
                k = torch.cat([kv, ka], 2).repeat_interleave(group, 1)
                v = torch.cat([vv, va], 2).repeat_interleave(group, 1)
                o = Fnn.scaled_dot_product_attention(q, k, v, attn_mask=mask)
                hv = _bf_branch_rest(mv.layers[l], hv, o[:, :, :P])
                ha = _bf_branch_rest(ma.layers[l], ha, o[:, :, P:])
            r = Fnn.rms_norm(ha, (d.hidden_a,), torch.tensor(head["final_norm"].astype(np.float64)), eps=d.rms_eps)
            vel = r @ torch.tensor(head["W_out"].astype(np.float64)).T + torch.tensor(head["b_out"].astype(np.float64))
        vels.append(vel.numpy())
        x = x - vel / steps
    return x.numpy(), vels


@pytest.mark.parametrize("P,S", [(5, 3), (64, 50)])
def test_cached_path_equals_brute_force_merged_sequence(tiny_weights, P, S):
    d = I.TINY.replace(chunk=S)
    w = I.Weights(d, seed=0, gain_jitter=0.1)
    emb = I.prefix_embeddings(d, 1, P)[0]
    x = I.noise(d, 1)[0]
    steps = 4
    chunk, vels = O.denoise(w, *O.prefill(w, emb)[:2], x, steps)
    chunk_bf, vels_bf = _brute_force_chunk(d, w, emb, x, steps)
    for a, b in zip(vels, vels_bf):
        assert np.max(np.abs(a - b)) <= 2e-5 * _rms(b)
    assert np.max(np.abs(chunk - chunk_bf)) <= 2e-5 * _rms(chunk_bf)


def test_merged_layer_equals_brute_force_single_layer():
    d = I.TINY
    w = I.Weights(d, seed=4, gain_jitter=0.1)
    P, S = 17, 50
    hp = I.hidden_states(P, d.hidden_v, seed=11)
    hs = I.hidden_states(S, d.hidden_a, seed=12)
    ov, oa, k, v = O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, hs, d)
    mv, ma = _qwen3(d, 0, w, layers=1), _qwen3(d, 1, w, layers=1)
    with torch.no_grad():
        qv, kv, vv = _bf_branch_qkv(mv.layers[0], mv.rotary_emb, torch.tensor(hp, dtype=torch.float64), np.arange(P))
        qa, ka, va = _bf_branch_qkv(ma.layers[0], ma.rotary_emb, torch.tensor(hs, dtype=torch.float64), np.arange(P, P + S))
        mask = torch.zeros(P + S, P + S, dtype=torch.bool)
        mask[:P, :P] = True
        mask[P:] = True
        g = d.n_q // d.n_kv
        o = Fnn.scaled_dot_product_attention(torch.cat([qv, qa], 2), torch.cat([kv, ka], 2).repeat_interleave(g, 1),
                                             torch.cat([vv, va], 2).repeat_interleave(g, 1), attn_mask=mask)
        rv = _bf_branch_rest(mv.layers[0], torch.tensor(hp, dtype=torch.float64), o[:, :, :P]).numpy()
        ra = _bf_branch_rest(ma.layers[0], torch.tensor(hs, dtype=torch.float64), o[:, :, P:]).numpy()
    assert np.max(np.abs(ov - rv)) <= 2e-5 * _rms(rv)
    assert np.max(np.abs(oa - ra)) <= 2e-5 * _rms(ra)
    assert np.max(np.abs(k - kv[0].numpy())) <= 2e-5 * _rms(k)
    # the library's RMSNorm runs in fp32 even for fp64 inputs
    assert np.max(np.abs(v - vv[0].numpy())) <= 2e-5 * _rms(v)


# ---------------------------------------------------------------- invariants of the method

def test_prefix_is_invariant_to_the_suffix():
    d = I.TINY
    w = I.Weights(d, seed=1)
    P = 20
    hp = I.hidden_states(P, d.hidden_v, seed=21)
    outs = [O.merged_layer(w.layer(0, 0), w.layer(1, 0), hp, I.hidden_states(S, d.hidden_a, seed=22 + S), d)
            for S in (3, 50)]
    for a, b in zip(outs[0][::2], outs[1][::2]):   # prefix output and K
        assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, _rms(a))
    np.testing.assert_allclose(outs[0][3], outs[1][3], rtol=0, atol=1e-12)
    # the suffix removed entirely: the prefill pass of a 1-layer model
    w1 = I.Weights(d.replace(layers=1), seed=1)
    ks, vs, h = O.prefill(w1, hp)
    assert np.max(np.abs(h - outs[0][0])) <= 1e-12 * _rms(h)
    assert np.max(np.abs(ks[0] - outs[0][2])) <= 1e-12


def test_zero_velocity_head_leaves_noise_unchanged():
    d = I.TINY
    w = I.Weights(d, seed=2)
    w.overrides[("head", "W_out")] = np.zeros((d.action_dim, d.hidden_a), np.float32)
    w.overrides[("head", "b_out")] = np.zeros(d.action_dim, np.float32)
    emb = I.prefix_embeddings(d, 1, 64)
    x = I.noise(d, 1)
    chunk, _, _ = O.infer(w, emb, x, steps=4)
    np.testing.assert_array_equal(chunk, x.astype(np.float64))


def test_constant_velocity_moves_by_minus_bias():
    d = I.TINY
    w = I.Weights(d, seed=2)
    c = np.linspace(-1, 1, d.action_dim).astype(np.float32)
    w.overrides[("head", "W_out")] = np.zeros((d.action_dim, d.hidden_a), np.float32)
    w.overrides[("head", "b_out")] = c
    emb = I.prefix_embeddings(d, 1, 64)
    x = I.noise(d, 1)
    chunk, _, _ = O.infer(w, emb, x, steps=5)
    np.testing.assert_allclose(chunk[0], x[0].astype(np.float64) - c.astype(np.float64)[None, :], rtol=0, atol=1e-12)


def test_closed_form_when_action_layers_write_nothing():
    """Wo = Wd = 0 in every action layer => h = e, so v = rms(e) W_out^T + b_out."""
    d = I.TINY
    w = I.Weights(d, seed=3, gain_jitter=0.1)
    for l in range(d.layers):
        w.overrides[(1, l, "Wo")] = np.zeros((d.hidden_a, d.n_q * d.head_dim), np.float32)
        w.overrides[(1, l, "Wd")] = np.zeros((d.hidden_a, d.inter_a), np.float32)
    emb = I.prefix_embeddings(d, 1, 64)
    x0 = I.noise(d, 1)
    steps = 4
    chunk, _, _ = O.infer(w, emb, x0, steps)
    hd = w.head()
    x = torch.tensor(x0[0].astype(np.float64))
    for kstep in range(steps):
        t = 1 - kstep / steps
        ang = t * 10000.0 ** (-torch.arange(d.hidden_a // 2) / (d.hidden_a // 2))
        e = x @ torch.tensor(hd["W_in"], dtype=torch.float64).T + torch.tensor(hd["b_in"], dtype=torch.float64) \
            + torch.cat([ang.sin(), ang.cos()])
        v = Fnn.rms_norm(e, (d.hidden_a,), torch.tensor(hd["final_norm"], dtype=torch.float64), eps=d.rms_eps) \
            @ torch.tensor(hd["W_out"], dtype=torch.float64).T + torch.tensor(hd["b_out"], dtype=torch.float64)
        x = x + (-1.0 / steps) * v
    np.testing.assert_allclose(chunk[0], x.numpy(), rtol=1e-12, atol=1e-12)


def test_batch_samples_are_independent():
    d = I.TINY
    w = I.Weights(d, seed=5)
    steps = 2
    emb2, x2 = I.prefix_embeddings(d, 2, 32), I.noise(d, 2)
    both, _, _ = O.infer(w, emb2, x2, steps)
    second, _, _ = O.infer(w, I.prefix_embeddings(d, 1, 32, seed=1001), I.noise(d, 1, seed=2001), steps)
    np.testing.assert_array_equal(both[1], second[0])


def test_generator_is_bf16_representable_and_seeded():
    d = I.TINY
    a = I.layer_weights(d, 1, 1, seed=0)
    b = I.layer_weights(d, 1, 1, seed=0)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    wq = a["Wq"]
    np.testing.assert_array_equal(I.round_bf16(wq), wq)
    assert abs(float(np.std(wq)) - 0.02) < 0.002
    # round-to-nearest-even on a few hand-checked values
    vals = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9], np.float32)
    np.testing.assert_array_equal(I.round_bf16(vals), np.array([1.0, 1.0 + 2.0 ** -6, 1.0], np.float32))
