"""Failure detection on the GPU without faulting it: a bounded wait that runs out.

Every pipeline wait of the library (TMA stage full/empty, accumulator ready,
softmax/MMA hand-offs) goes through one bounded mbarrier wait.  The self-test
kernel waits on an mbarrier that nothing arrives on; the wait must give up
after its limit, record the timeout in the device error word and return, so
that the host sees DM0_EDEVICE, the context stays usable and dm0_clear_error
restores it.  No trap, no assert, no bad address, no endless loop.
"""
import time

import numpy as np
import pytest
import torch

from synth import inputs as I
from tests.gpu_util import rel_err, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_recovers():
    from oracle import dm0_oracle as O
    from vla_dual_expert_b200 import Dm0Error, Engine, build
    build.build()
    d = I.TINY
    w = I.Weights(d, seed=0)
    eng = Engine(d, 1, 64)
    try:
        eng.load_from(w)
        assert eng.device_error() == 0
        t0 = time.perf_counter()
        eng.selftest_timeout(limit_us=20000)        # 20 ms
        with pytest.raises(Dm0Error) as e:
            eng.sync()
        elapsed = time.perf_counter() - t0
        assert e.value.status == -5                  # DM0_EDEVICE
        assert eng.device_error() & 1
        assert 0.015 < elapsed < 5.0                 # it waited its limit, then gave up
        eng.clear_error()
        assert eng.device_error() == 0
        # the context still computes correct results
        emb, noise = I.prefix_embeddings(d, 1, 64), I.noise(d, 1)
        eng.prefill(to_dev_bf16(emb))
        out = eng.denoise(to_dev_f32(noise), 4)
        eng.sync()
        ref, _, _ = O.infer(w, emb, noise, 4)
        assert rel_err(out.cpu().numpy(), ref) <= 2e-2
    finally:
        eng.close()


def test_selftest_rejects_bad_limit():
    from vla_dual_expert_b200 import Dm0Error, Engine
    eng = Engine(I.TINY, 1, 64)
    try:
        with pytest.raises(Dm0Error) as e:
            eng.selftest_timeout(limit_us=0)
        assert e.value.status == -2
    finally:
        eng.close()
