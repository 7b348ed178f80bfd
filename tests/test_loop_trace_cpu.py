"""The phase-timeline summary of the single-launch Euler loop (bench.py --b1-trace) on a synthetic
trace: per-phase medians over the CTAs (the attention phase over its item CTAs only), the operand
copies' time in flight, and each phase's wall time from its latest start to the next phase's."""
import numpy as np

import bench


def _synthetic(layers=2, steps=1, ctas=6, items=2):
    """Phase q starts at 10 q us, CTA j 0.1 j us late; marks 1, 2, 3, 5 at +1, +2, +3, +4 us from the
    start (attention items twice as slow), copies issued at +0.5 and landed at +0.7."""
    per_step = 5 * layers + 1
    rows = 1 + steps * per_step
    arr = np.zeros((rows, ctas, bench.TRACE_SLOTS))
    for q in range(rows):
        rr = (q - 1) % per_step
        att = q >= 1 and rr < 5 * layers and rr % 5 == 1
        for c in range(ctas):
            start = 10.0 * q + 0.1 * c
            slow = 2.0 if (att and c < items) else 1.0
            arr[q, c, 0] = start
            for sl, off in ((1, 1.0), (2, 2.0), (3, 3.0), (5, 4.0)):
                arr[q, c, sl] = start + off * slow
            arr[q, c, 8] = start + 0.5
            arr[q, c, 9] = start + 0.7
    return arr * 1000.0


def test_summary_medians_and_phase_time():
    out = bench.summarize_loop_trace(_synthetic(steps=2), layers=2, items=2)
    assert set(out) == {"qkv", "attention", "o_proj", "gate_up", "down", "step"}
    q = out["qkv"]
    assert (q["staged"], q["acc_ready"], q["issued"], q["arrived"]) == (1.0, 2.0, 3.0, 4.0)
    assert abs(q["copies"] - 0.2) < 1e-9
    assert abs(q["phase"] - 10.0) < 1e-9          # latest start to the next phase's latest start
    assert abs(q["last_arrival"] - 4.0) < 1e-9    # the latest CTA also starts latest
    a = out["attention"]                           # only the two item CTAs, which run 2x slower
    assert (a["staged"], a["issued"], a["arrived"]) == (2.0, 6.0, 8.0)
    assert set(out["step"]) == {"phase"}
