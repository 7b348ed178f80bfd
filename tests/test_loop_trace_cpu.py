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
    assert abs(q["to_copies"] - 0.5) < 1e-9      # copies issued 0.5 us after the start
    assert abs(q["build"] - 0.3) < 1e-9          # landed at +0.7, staged at +1.0
    assert abs(q["phase"] - 10.0) < 1e-9          # latest start to the next phase's latest start
    assert abs(q["last_arrival"] - 4.0) < 1e-9    # the latest CTA also starts latest
    a = out["attention"]                           # only the two item CTAs, which run 2x slower
    assert (a["staged"], a["issued"], a["arrived"]) == (2.0, 6.0, 8.0)
    assert set(out["step"]) == {"phase"}


def test_gemm_trace_summary():
    """bench.summarize_gemm_trace on a synthetic two-launch trace: the shape words of CTA 0, the
    CTAs that ran (stale rows and unused slots ignored), the span from the first entry to the last
    exit, per-mark medians from the first entry, and the last tile's epilogue of one-tile CTAs taken
    from their first tile."""
    ctas, slots = 6, bench.GEMM_TRACE_SLOTS
    arr = np.zeros((3, ctas, slots), dtype=np.uint64)
    base = 5_000_000_000
    for c in range(4):   # launch 0: 4 CTAs ran, each 1 us later than the previous
        t = base + 1000 * c
        arr[0, c, :10] = [t + 1000 * m for m in range(10)]
        if c < 2:        # CTAs 0 and 1 had one tile: no "last_done" mark
            arr[0, c, 7] = 0
    arr[0, 4, :10] = 7   # a stale row from long before: not part of the launch
    arr[0, 0, 14] = (816 << 32) | 4096
    arr[0, 0, 15] = (2048 << 32) | 256
    arr[1, 0, :10] = [base + 50_000_000 + 2000 * m for m in range(10)]   # launch 1: one CTA
    arr[1, 0, 14] = (50 << 32) | 128
    arr[1, 0, 15] = (64 << 32) | 64
    # QKV epilogue SM-cycle marks (slots 10-13) on launch 0: the RMS pass 1000 + 100 c cycles, the RoPE
    # pass 5000, the tile 14000; CTA 3 has no marks (a V-only tile) and is left out of them
    for c in range(3):
        c0 = 1_000_000 * (c + 1)
        arr[0, c, 10:14] = [c0, c0 + 1000 + 100 * c, c0 + 6000 + 100 * c, c0 + 14000]
    out = bench.summarize_gemm_trace(arr)
    assert len(out) == 2
    a, b = out
    assert (a["M"], a["N"], a["K"], a["BN"], a["ctas"]) == (816, 4096, 2048, 256, 4)
    assert a["span_us"] == 12.0            # last exit (CTA 3: +3 + 9 us) after the first entry
    assert a["setup"] == 2.5               # median over CTAs of (1 us + their 0..3 us delay)
    assert a["last_done"] == 8.0           # one-tile CTAs count their first tile: 6, 7, 9, 10
    assert a["qkv_epi_kcycles"] == {"rms_pass": 1.1, "rope_pass": 5.0, "tile": 14.0}
    assert (b["ctas"], b["span_us"], b["exit"]) == (1, 18.0, 18.0)
    assert "qkv_epi_kcycles" not in b


def test_attn_trace_summary():
    """bench.summarize_attn_trace on a synthetic trace: every CTA announces P of block j at 2 us j +
    1.6 us, sees S 0.5 us after the MMA warp issued it, and exchanges the max 0.4 us later; a CTA with a
    missing stamp is left out."""
    arr = np.zeros((5, 64, 4), dtype=np.uint64)
    for c in range(4):
        for j in range(10):
            base = 1_000_000 + 100 * c + 2000 * j
            arr[c, j] = [base + 500, base + 900, base + 1600, base]
    arr[4, :10] = 7
    arr[4, 3, 2] = 0
    out = bench.summarize_attn_trace(arr, 10)
    assert out["ctas"] == 4
    assert (out["period"], out["wait_for_s"], out["s_to_max"], out["max_to_p"], out["s_issue_lead"]) == \
        (2.0, 0.9, 0.4, 0.7, 0.5)
    assert out["walk_us"] == 19.1
