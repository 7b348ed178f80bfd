"""Tolerances of the GPU parity tests, in one place.

Two kinds:
  * the stated bars: max |gpu - oracle| <= 1e-2 RMS(oracle) for one merged layer on identical fp32
    inputs, and <= 2e-2 RMS for the final action chunk (per-step velocities of a shallow model are held
    to the chunk's 2e-2 of RMS(v));
  * depth-dependent bars, where bf16 roundings of many layers add up: each is twice the error that
    the CPU emulation of the GPU's bf16 rounding points (tests/bf16_emulation.py) shows on the same
    seeded inputs, rounded up.  tests/test_tolerance_emulation_cpu.py recomputes the emulation and
    fails if any bar here leaves less than that factor of two.

bf16-stored tensors (K/V, attention output) are compared element-wise with
|d_i| <= a RMS(ref) + 2^-8 |ref_i| and RMS(d) <= r RMS(ref) (tests/gpu_util.check_bf16): the 2^-8 |ref_i|
term is the rounding of the stored bf16 value itself (2^-9 relative), doubled.
"""

# ------------------------------------------------------------------ stated bars
LAYER = 1e-2        # one merged layer: fp32 residual outputs of both branches
CHUNK = 2e-2        # final action chunk; per-step velocities of the 2- and 3-layer models
KV_ONE_LAYER = (1e-2, 5e-3)   # (a, r): the K/V of one layer (the layer bar plus the storage rounding)
ATTN_OUT = (2e-2, 5e-3)       # (a, r): one attention call on bf16 inputs (P is also rounded before PV)

# ------------------------------------------------------------------ derived from the bf16 emulation
# (a, r) of the K/V cache of prefill layer l, DM0-base widths, one 816-token prefix (seed 1000):
# emulated RMS(d) 1.7e-3 / 7.0e-3 / 9.9e-3 of RMS at layers 0 / 13 / 27
KV_DEPTH_DM0 = {0: (1.6e-2, 3.5e-3), 13: (8.0e-2, 1.5e-2), 27: (1.1e-1, 2.0e-2)}
# (a, r) of every layer's K/V of the 2-layer tiny model at P = 64 and 37 (emulated RMS(d) <= 2.4e-3)
KV_TINY = (1.7e-2, 5.0e-3)
# velocity at the top of the 28-layer action stack over an 816-token cache, every step:
# (RMS(d), max |d|) / RMS(v); emulated <= 4.7e-3 and 1.9e-2
VEL_STACK = (1.0e-2, 4.0e-2)
# the FP8 VLM MLP inside one full-width merged layer (P = 816 and 333, seeds 40.., gain jitter 0.1):
# RMS(d) / RMS of the VLM output against the FP8 oracle; emulated 1.11e-2 .. 1.26e-2
FP8_LAYER_RMS = 2.6e-2
# every layer's K/V of the tiny model's FP8 prefix pass (P = 64): RMS(d) / RMS; emulated <= 2.5e-3
FP8_TINY_KV_RMS = 5.0e-3
