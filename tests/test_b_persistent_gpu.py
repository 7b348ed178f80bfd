"""The single-launch persistent Euler loop (one observation, head_dim 128): the action chunk and every
step's velocity against the fp64 oracle, and against the per-layer kernel path of the same context.

DM0-base widths with 3 layers keep the oracle fast; the 28-layer stack goes through the same kernel
in test_a_gpu_parity (denoise over a random cache, and end to end).  Prefix lengths cover a whole
number of 64-key blocks (64), a ragged last block (100, 816) and a single key (1); the key-split
count per KV head is varied from 1 (one CTA per head walks every block) to 8.

Tolerances as in test_a_gpu_parity: chunk 2e-2 of RMS(chunk), velocities 2e-2 of RMS(v) for this
shallow stack.  The two GPU paths differ only in fp32 summation order (split-K partial sums reach
the accumulators in a different order), so they agree to 1e-2 of RMS."""
import os

import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O
from synth import inputs as I
from tests.gpu_util import device_view_bf16, host, rel_err, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

STEPS = 3


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from vla_dual_expert_b200 import build
    build.build()


@pytest.fixture(scope="module")
def small():
    d = I.DM0_BASE.replace(layers=3)
    return d, I.Weights(d, seed=0, gain_jitter=0.1)


def _engine(d, w, env, max_prefix=816):
    """Engine created while `env` is set (the loop selection is read when the context is created)."""
    from vla_dual_expert_b200 import Engine
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        eng = Engine(d, 1, max_prefix)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    eng.load_from(w)
    return eng


def _load_random_cache(eng, d, P):
    kp, vp = eng.kv_view()
    n = d.layers * d.n_kv * P * d.head_dim
    shape = (d.layers, 1, d.n_kv, P, d.head_dim)
    kc, vc = device_view_bf16(kp, (n,)).view(shape), device_view_bf16(vp, (n,)).view(shape)
    ks, vs = [], []
    for l in range(d.layers):
        k, v = I.random_kv_layer(d, 1, P, l)
        kc[l].copy_(to_dev_bf16(k))
        vc[l].copy_(to_dev_bf16(v))
        ks.append(k[0].astype(np.float64))
        vs.append(v[0].astype(np.float64))
    eng.kv_commit(1, P)
    return ks, vs


def _run(eng, d, noise):
    vel = torch.empty((STEPS, 1, d.chunk, d.action_dim), device="cuda", dtype=torch.float32)
    n0 = eng.launch_count()
    chunk = eng.denoise(to_dev_f32(noise), STEPS, velocities=vel)
    eng.sync()
    return host(chunk[0]), host(vel[:, 0]), eng.launch_count() - n0


@pytest.mark.parametrize("P,splits", [(816, "4"), (816, "1"), (816, "8"), (100, "3"), (64, "2"), (1, "4")])
def test_persistent_loop_matches_oracle(small, P, splits):
    d, w = small
    eng = _engine(d, w, {"DM0_PERSIST_SPLITS": splits})
    try:
        ks, vs = _load_random_cache(eng, d, P)
        noise = I.noise(d, 1)
        chunk, vel, launches = _run(eng, d, noise)
        assert launches == 1, "the Euler loop should be one kernel launch"
        ref, ref_v = O.denoise(w, ks, vs, noise[0], STEPS)
        for k in range(STEPS):
            assert rel_err(vel[k], ref_v[k]) <= 2e-2, f"velocity step {k}"
        assert rel_err(chunk, ref) <= 2e-2
    finally:
        eng.close()


def test_persistent_loop_matches_per_layer_kernels(small):
    d, w = small
    P = 816
    eng_p = _engine(d, w, {})
    eng_k = _engine(d, w, {"DM0_NO_PERSIST": "1"})
    try:
        _load_random_cache(eng_p, d, P)
        _load_random_cache(eng_k, d, P)
        noise = I.noise(d, 1)
        cp, vp, lp = _run(eng_p, d, noise)
        ck, vk, lk = _run(eng_k, d, noise)
        assert lp == 1 and lk == 1 + STEPS * (5 * d.layers + 1)
        assert rel_err(cp, ck) <= 1e-2
        for k in range(STEPS):
            assert rel_err(vp[k], vk[k]) <= 1e-2, f"velocity step {k}"
    finally:
        eng_p.close()
        eng_k.close()


def test_persistent_loop_repeat_and_step_count_change(small):
    """Back-to-back calls (scratch left clean by the previous launch), including a different K.
    Repeated runs are not bitwise equal: split-K partial sums reach the fp32 accumulators in
    arrival order, and a changed last bit can flip a later bf16 rounding of an activation, so
    repeats are held to the same 1e-2 as the two GPU paths."""
    d, w = small
    eng = _engine(d, w, {})
    try:
        ks, vs = _load_random_cache(eng, d, 816)
        noise = I.noise(d, 1)
        first, _, _ = _run(eng, d, noise)
        short = host(eng.denoise(to_dev_f32(noise), 1)[0])
        again, _, _ = _run(eng, d, noise)
        eng.sync()
        assert rel_err(again, first) <= 1e-2
        ref1, _ = O.denoise(w, ks, vs, noise[0], 1)
        assert rel_err(short, ref1) <= 2e-2
        assert eng.device_error() == 0
    finally:
        eng.close()
