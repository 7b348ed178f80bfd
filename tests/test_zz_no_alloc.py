"""The allocation-free attention entry point (dm0_attention_noalloc).

Some callers of this library cannot call cudaMalloc once they are running: a
robot's real-time control loop, code inside CUDA stream capture, or a host
whose device memory belongs to another allocator.  dm0_attention_noalloc serves
them: it takes only inputs and outputs and keeps its split-KV scratch in a
fixed array inside the library.  This test calls it through the C ABI twice in
a row and checks each result element by element against the oracle's attention
and against dm0_op_attention (the context-based entry point, whose scratch comes
from cudaMalloc) on the same inputs, with the attention tolerance the other GPU
tests use.  It is self-contained so that it passes when run alone in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import dm0_oracle as O
from synth import inputs as I
from tests.gpu_util import check_bf16, host, to_dev_bf16

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Tq, Ta, Tb, d):
    rng = np.random.default_rng(seed)
    bf = lambda *s: I.round_bf16(rng.standard_normal(s).astype(np.float32))
    D = d.head_dim
    return (bf(B, Tq, d.n_q, D), bf(B, d.n_kv, Ta, D), bf(B, d.n_kv, Ta, D), bf(B, d.n_kv, Tb, D),
            bf(B, d.n_kv, Tb, D))


def test_noalloc_attention_matches_context_entry_point():
    assert torch.cuda.is_available()
    from vla_dual_expert_b200 import Engine, build, load_library
    build.build()
    lib = load_library()
    d = I.DM0_BASE.replace(layers=1)
    B, Tq, Ta, Tb, splits = 1, 50, 816, 50, 4      # the batch-1 suffix attention: 8 groups x 4 splits = 32 slots
    eng = Engine(d, B, Ta)
    try:
        for call, seed in enumerate((11, 12)):
            host_in = _inputs(seed, B, Tq, Ta, Tb, d)
            q, ka, va, kb, vb = (to_dev_bf16(x) for x in host_in)
            ref = torch.full(q.shape, float("nan"), device="cuda", dtype=torch.bfloat16)
            eng.op_attention(q, ka, va, kb, vb, ref, splits=splits)
            out = torch.full(q.shape, float("nan"), device="cuda", dtype=torch.bfloat16)
            stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            st = lib.dm0_attention_noalloc(q.data_ptr(), ka.data_ptr(), va.data_ptr(), Ta, kb.data_ptr(),
                                           vb.data_ptr(), Tb, out.data_ptr(), B, Tq, d.n_q, d.n_kv, d.head_dim,
                                           splits, stream)
            assert st == 0, f"call {call}: status {st}"
            torch.cuda.synchronize()
            hq, hka, hva, hkb, hvb = (x.astype(np.float64) for x in host_in)
            for b in range(B):   # every query row sees all Ta + Tb keys
                want = O.attention(hq[b].transpose(1, 0, 2), np.concatenate([hka[b], hkb[b]], axis=1),
                                   np.concatenate([hva[b], hvb[b]], axis=1),
                                   np.ones((Tq, Ta + Tb), dtype=bool)).transpose(1, 0, 2)
                check_bf16(host(out[b]), want, 2e-2, f"no-alloc call {call} vs the oracle")
            check_bf16(host(out), host(ref), 2e-2, f"no-alloc call {call} vs dm0_op_attention")
        # a split count beyond the fixed scratch is rejected, not run
        big = to_dev_bf16(_inputs(13, 2, Tq, Ta, Tb, d)[0])
        st = lib.dm0_attention_noalloc(big.data_ptr(), ka.data_ptr(), va.data_ptr(), Ta, kb.data_ptr(),
                                       vb.data_ptr(), Tb, big.data_ptr(), 2, Tq, d.n_q, d.n_kv, d.head_dim, 14,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == -2
    finally:
        eng.close()
