"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module holds shapes, seeds and random draws only: it performs none of
the model's arithmetic.  Every tensor is drawn from its own counter-seeded
PCG64 stream, so any single layer can be generated on its own (the CPU
oracle never has to materialise a full 28-layer model to check one layer).

Shapes follow the DM0-base configuration on the DM0 architecture notes page
(dregs-remover.com/news/27019, section 1): 28+28 Qwen3 layers, VLM hidden
2048, action-expert hidden 1024, 16 query heads, 8 KV heads, head_dim 128,
action dim 32, chunk 50.  Intermediate sizes (6144 / 3072), RoPE theta 1e6
and the N(0, 0.02) weight / N(0, 1) embedding and noise distributions are the
workload definitions this library is measured on.

Matrices are returned as float32 arrays whose values are exactly
representable in bfloat16 (round-to-nearest-even of an fp32 draw): the GPU
stores them as bf16 and the oracle upcasts the same values, so both sides see
identical parameters.  Norm gains and biases stay float32.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

# tensor order inside one decoder layer (also the blob order)
LAYER_TENSORS = ("attn_norm", "Wq", "Wk", "Wv", "q_norm", "k_norm",
                 "Wo", "mlp_norm", "Wg", "Wu", "Wd")
HEAD_TENSORS = ("W_in", "b_in", "final_norm", "W_out", "b_out")
# time-modulated action expert (DM0.5): the time MLP and the final norm's modulator ...
TIME_TENSORS = ("W_ti", "b_ti", "W_to", "b_to", "W_mf", "b_mf")
# ... and one modulator per action layer for each of its two pre-norms (attention, MLP)
MOD_TENSORS = ("W_ma", "b_ma", "W_mm", "b_mm")
BRANCH_VLM, BRANCH_ACTION = 0, 1


@dataclass(frozen=True)
class Dims:
    layers: int
    hidden_v: int
    inter_v: int
    hidden_a: int
    inter_a: int
    n_q: int
    n_kv: int
    head_dim: int
    chunk: int = 50
    action_dim: int = 32
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6

    def hidden(self, branch: int) -> int:
        return self.hidden_v if branch == BRANCH_VLM else self.hidden_a

    def inter(self, branch: int) -> int:
        return self.inter_v if branch == BRANCH_VLM else self.inter_a

    def replace(self, **kw) -> "Dims":
        return dataclasses.replace(self, **kw)


# DM0-base shapes (28-layer Qwen3 VLM hidden 2048 + 28-layer Qwen3 action expert hidden 1024)
DM0_BASE = Dims(layers=28, hidden_v=2048, inter_v=6144, hidden_a=1024, inter_a=3072,
                n_q=16, n_kv=8, head_dim=128)
# tiny merged-attention model: 2 layers, hidden 256/128, 4 q / 2 kv heads of 32
TINY = Dims(layers=2, hidden_v=256, inter_v=512, hidden_a=128, inter_a=256,
            n_q=4, n_kv=2, head_dim=32)


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    batch: int
    prefix: int          # P prefix tokens per sample
    steps: int           # Euler steps K
    random_kv: bool = False  # denoise over an injected random bf16 KV cache


WORKLOADS = {
    # 2 layers, P=64, S=50, 4 Euler steps, fp32-sized toy
    "tiny": Workload("tiny", TINY, batch=1, prefix=64, steps=4),
    # one full-width merged layer, P=816 (3 views x 256 image tokens + 48 text tokens)
    "merged_layer": Workload("merged_layer", DM0_BASE.replace(layers=1), batch=1, prefix=816, steps=0),
    # 28-layer action expert over a random bf16 prefix KV cache, 10 steps, batch 1
    "denoise_b1": Workload("denoise_b1", DM0_BASE, batch=1, prefix=816, steps=10, random_kv=True),
    # prefill (P=816) + 10-step denoise at batch 1
    "e2e_b1": Workload("e2e_b1", DM0_BASE, batch=1, prefix=816, steps=10),
    # batch 16, P=2048 each, 10 steps
    "e2e_b16": Workload("e2e_b16", DM0_BASE, batch=16, prefix=2048, steps=10),
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


_CHUNK = 1 << 20
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        import concurrent.futures
        import os
        _POOL = concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1))
    return _POOL


def _fill(out: np.ndarray, entropy: tuple, c: int, scale: float, bf16: bool):
    lo = c * _CHUNK
    part = out[lo:lo + _CHUNK]
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(entropy) + [c])))
    rng.standard_normal(size=part.shape, dtype=np.float32, out=part)
    if scale != 1.0:
        part *= np.float32(scale)
    if bf16:
        part[...] = round_bf16(part)


def _normal(entropy: tuple, shape, scale: float = 1.0, bf16: bool = False) -> np.ndarray:
    """N(0, scale^2) fp32 draw; element chunk c (2^20 elements) comes from its own
    PCG64 stream seeded by (entropy..., c), so the result does not depend on
    how many threads fill it.  bf16=True rounds every value to bf16 (RNE)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    chunks = (n + _CHUNK - 1) // _CHUNK
    if chunks <= 1:
        _fill(out, entropy, 0, scale, bf16)
    else:
        list(_pool().map(lambda c: _fill(out, entropy, c, scale, bf16), range(chunks)))
    return out.reshape(shape)


def layer_shapes(d: Dims, branch: int) -> dict:
    H, I, D = d.hidden(branch), d.inter(branch), d.head_dim
    return {
        "attn_norm": (H,), "Wq": (d.n_q * D, H), "Wk": (d.n_kv * D, H), "Wv": (d.n_kv * D, H),
        "q_norm": (D,), "k_norm": (D,), "Wo": (H, d.n_q * D), "mlp_norm": (H,),
        "Wg": (I, H), "Wu": (I, H), "Wd": (H, I),
    }


def head_shapes(d: Dims) -> dict:
    return {"W_in": (d.hidden_a, d.action_dim), "b_in": (d.hidden_a,),
            "final_norm": (d.hidden_a,), "W_out": (d.action_dim, d.hidden_a),
            "b_out": (d.action_dim,)}


def _gain(entropy, shape, jitter):
    if jitter == 0.0:
        return np.ones(shape, dtype=np.float32)
    return (1.0 + _normal(entropy, shape, jitter)).astype(np.float32)


def layer_weights(d: Dims, branch: int, layer: int, seed: int = 0,
                  std: float = 0.02, gain_jitter: float = 0.0) -> dict:
    """Parameters of one decoder layer of one branch (VLM=0, action expert=1).

    Matrices are [out][in] and bf16-representable; norm gains are 1, or
    1 + gain_jitter * N(0,1) when gain_jitter > 0.
    """
    out = {}
    for tid, (name, shape) in enumerate(layer_shapes(d, branch).items()):
        ent = (seed, branch, layer, tid)
        if name.endswith("norm"):
            out[name] = _gain(ent, shape, gain_jitter)
        else:
            out[name] = _normal(ent, shape, std, bf16=True)
    return out


def head_weights(d: Dims, seed: int = 0, std: float = 0.02, gain_jitter: float = 0.0) -> dict:
    """action_in_proj (W_in, b_in), final RMSNorm gain, action_out_proj (W_out, b_out)."""
    out = {}
    for tid, (name, shape) in enumerate(head_shapes(d).items()):
        ent = (seed, 2, 0, tid)
        if name == "final_norm":
            out[name] = _gain(ent, shape, gain_jitter)
        elif name.startswith("W"):
            out[name] = _normal(ent, shape, std, bf16=True)
        else:
            out[name] = _normal(ent, shape, std)
    return out


def time_shapes(d: Dims) -> dict:
    H = d.hidden_a
    return {"W_ti": (H, H), "b_ti": (H,), "W_to": (H, H), "b_to": (H,),
            "W_mf": (2 * H, H), "b_mf": (2 * H,)}


def mod_shapes(d: Dims) -> dict:
    H = d.hidden_a
    return {"W_ma": (3 * H, H), "b_ma": (3 * H,), "W_mm": (3 * H, H), "b_mm": (3 * H,)}


def _draw_group(shapes: dict, ent0: tuple, std: float) -> dict:
    """Matrices N(0, std^2) rounded to bf16; vectors (biases) N(0, std^2) fp32."""
    return {name: _normal(ent0 + (tid,), shape, std, bf16=len(shape) == 2)
            for tid, (name, shape) in enumerate(shapes.items())}


def time_weights(d: Dims, seed: int = 0, std: float = 0.02) -> dict:
    """time_mlp_in (W_ti, b_ti), time_mlp_out (W_to, b_to) and the final norm's modulator (W_mf, b_mf)."""
    return _draw_group(time_shapes(d), (seed, 4, 0), std)


def mod_weights(d: Dims, layer: int, seed: int = 0, std: float = 0.02) -> dict:
    """The two time modulators of action layer `layer`: attention pre-norm (W_ma, b_ma), MLP pre-norm
    (W_mm, b_mm); each maps the time condition to three vectors of hidden_a."""
    return _draw_group(mod_shapes(d), (seed, 3, layer), std)


class Weights:
    """Lazily generated model parameters (per-layer access, cached on request)."""

    def __init__(self, d: Dims, seed: int = 0, std: float = 0.02, gain_jitter: float = 0.0,
                 cache: bool = True):
        self.d, self.seed, self.std, self.gain_jitter = d, seed, std, gain_jitter
        self._cache = {} if cache else None
        self._head = None
        self._time = None
        self._mods = {} if cache else None
        # (branch, layer, name), ("head", name), ("time", name) or ("mod", layer, name) -> array
        self.overrides = {}

    def layer(self, branch: int, layer: int) -> dict:
        key = (branch, layer)
        if self._cache is not None and key in self._cache:
            w = self._cache[key]
        else:
            w = layer_weights(self.d, branch, layer, self.seed, self.std, self.gain_jitter)
            if self._cache is not None:
                self._cache[key] = w
        if any(k[:2] == key for k in self.overrides if len(k) == 3 and k[0] != "mod"):
            w = dict(w)
            for k, v in self.overrides.items():
                if len(k) == 3 and k[:2] == key:
                    w[k[2]] = v
        return w

    def _with_overrides(self, w: dict, key: tuple) -> dict:
        extra = {k[-1]: v for k, v in self.overrides.items() if k[:-1] == key}
        return dict(w, **extra) if extra else w

    def time(self) -> dict:
        """Time MLP and final-norm modulator of the time-modulated action expert."""
        if self._time is None:
            self._time = time_weights(self.d, self.seed, self.std)
        return self._with_overrides(self._time, ("time",))

    def mod(self, layer: int) -> dict:
        """Time modulators of action layer `layer`."""
        if self._mods is not None and layer in self._mods:
            w = self._mods[layer]
        else:
            w = mod_weights(self.d, layer, self.seed, self.std)
            if self._mods is not None:
                self._mods[layer] = w
        return self._with_overrides(w, ("mod", layer))

    def head(self) -> dict:
        if self._head is None:
            self._head = head_weights(self.d, self.seed, self.std, self.gain_jitter)
        w = self._head
        if any(k[0] == "head" for k in self.overrides):
            w = dict(w)
            for k, v in self.overrides.items():
                if k[0] == "head":
                    w[k[1]] = v
        return w


def prefix_embeddings(d: Dims, batch: int, prefix: int, seed: int = 1000) -> np.ndarray:
    """[B][P][hidden_v] N(0,1) prefix embeddings, bf16-representable (sample b uses seed+b)."""
    return np.stack([_normal((seed + b,), (prefix, d.hidden_v), bf16=True) for b in range(batch)])


def noise(d: Dims, batch: int, seed: int = 2000) -> np.ndarray:
    """[B][chunk][action_dim] N(0,1) fp32 initial x_1 (sample b uses seed+b)."""
    return np.stack([_normal((seed + b,), (d.chunk, d.action_dim)) for b in range(batch)])


def random_kv_layer(d: Dims, batch: int, prefix: int, layer: int, seed: int = 3000):
    """bf16-representable N(0,1) K and V of one layer: each [B][n_kv][P][head_dim]."""
    k = np.stack([_normal((seed + b, layer, 0), (d.n_kv, prefix, d.head_dim), bf16=True)
                  for b in range(batch)])
    v = np.stack([_normal((seed + b, layer, 1), (d.n_kv, prefix, d.head_dim), bf16=True)
                  for b in range(batch)])
    return k, v


def hidden_states(batch_tokens: int, hidden: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """fp32 N(0, scale^2) residual-stream inputs for single-layer checks."""
    return _normal((seed, 7), (batch_tokens, hidden), scale)


def train_batch(d: Dims, batch: int, seed: int = 4000):
    """Synthetic flow-matching training inputs, sample b from seed + b.

    actions a and noise eps: [B][chunk][action_dim] N(0, 1) fp32; t: [B] uniform in [0, 1) (float64);
    mask: [B][chunk][action_dim] bool marking the valid entries: the first n_dims action dimensions
    (a robot whose action vector is shorter than action_dim, zero-padded) of the first n_steps chunk
    positions (an episode that ends inside the chunk), n_dims uniform in [1, action_dim] and n_steps
    uniform in [1, chunk].
    """
    a, eps, t, mask = [], [], [], []
    for b in range(batch):
        a.append(_normal((seed + b, 0), (d.chunk, d.action_dim)))
        eps.append(_normal((seed + b, 1), (d.chunk, d.action_dim)))
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed + b, 2])))
        t.append(rng.random())
        n_dims = int(rng.integers(1, d.action_dim + 1))
        n_steps = int(rng.integers(1, d.chunk + 1))
        m = np.zeros((d.chunk, d.action_dim), dtype=bool)
        m[:n_steps, :n_dims] = True
        mask.append(m)
    return np.stack(a), np.stack(eps), np.asarray(t, np.float64), np.stack(mask)
