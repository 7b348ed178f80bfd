"""The phase-timeline reader of the persistent Euler loop (vla_dual_expert_b200/loop_trace.py) on a
synthetic trace: per-phase medians, the phase wall time from one phase's latest start to the next,
and the attention phase restricted to its item CTAs."""
import numpy as np

from vla_dual_expert_b200 import loop_trace


def _synthetic(layers=2, steps=1, ctas=6, items=2):
    """Each phase starts 10 us after the previous; a CTA's marks sit at fixed offsets from its start,
    every CTA j starts j * 0.1 us late; attention items are slower (offset x 2)."""
    nph = 1 + steps * (5 * layers + 1)
    arr = np.zeros((nph, ctas, loop_trace.SLOTS))
    per_step = 5 * layers + 1
    for q in range(nph):
        for c in range(ctas):
            start = 10.0 * q + 0.1 * c
            r = (q - 1) % per_step
            slow = 2.0 if (q >= 1 and r < 5 * layers and r % 5 == 1 and c < items) else 1.0
            arr[q, c, 0] = start
            arr[q, c, 1] = start + 1.0 * slow
            arr[q, c, 2] = start + 2.0 * slow
            arr[q, c, 3] = start + 3.0 * slow
            arr[q, c, 5] = start + 4.0 * slow
    return arr


def test_summary_medians_and_phase_time():
    arr = _synthetic(steps=2)   # the last phase has no successor, so a step boundary needs two steps
    out = loop_trace.summarize(arr, layers=2, attention_ctas=2)
    assert set(out) == {"qkv", "attention", "o_proj", "gate_up", "down", "step"}
    q = out["qkv"]
    assert (q["staged"], q["acc_ready"], q["issued"], q["arrived"]) == (1.0, 2.0, 3.0, 4.0)
    assert q["phase"] == 10.0                      # latest start to latest start of the next phase
    assert abs(q["last_arrival"] - 4.0) < 1e-9     # the latest CTA also starts latest
    a = out["attention"]                           # only the two item CTAs, which run 2x slower
    assert (a["staged"], a["issued"], a["arrived"]) == (2.0, 6.0, 8.0)
    assert set(out["step"]) == {"phase"}


def test_phase_names_follow_the_schedule():
    # phase 0 is the input of step 0; then 5 phases per layer and one step boundary per step; the
    # final step boundary has no next phase and is not summarised
    out1 = loop_trace.summarize(_synthetic(layers=3, steps=1), layers=3, attention_ctas=2)
    assert "step" not in out1 and out1["down"]["phase"] == 10.0
    out2 = loop_trace.summarize(_synthetic(layers=3, steps=2), layers=3, attention_ctas=2)
    assert out2["step"]["phase"] == 10.0
