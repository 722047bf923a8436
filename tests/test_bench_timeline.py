"""bench.py's reduction of the step kernel's timeline stamps to per-phase critical-path times
(CPU only): a synthetic 3-CTA, 2-layer timeline with known phase and barrier durations."""

import numpy as np

import bench


def synthetic_timeline(L, ncta, work_ns, release_ns, skew_ns):
    """Stamps in the kernel's order (bench.timeline_names): CTA c arrives c * skew_ns after CTA 0
    at every barrier; every CTA leaves a barrier release_ns after the last arrival; staging and
    the intermediate stamps take 0 ns."""
    names = bench.timeline_names(L)
    rows = np.zeros((ncta, len(names)), dtype=np.int64)
    t = 0
    cur = "qkv"
    for k, name in enumerate(names):
        if name == "start":
            continue
        parts = name.split(".")
        kind = parts[-1]
        if kind == "arrive":
            t += work_ns[cur]
            for c in range(ncta):
                rows[c, k] = t + c * skew_ns
            t += (ncta - 1) * skew_ns
            cur = parts[-2] if parts[0] != "head" else "head"
        elif kind == "exit":
            t += release_ns
            rows[:, k] = t
        elif name == "end":
            t += work_ns["head"]
            rows[:, k] = t
        else:
            rows[:, k] = t
    return rows


def test_phase_breakdown_recovers_known_durations():
    L, ncta, release, skew = 2, 3, 700, 40
    work = {"qkv": 1000, "attn": 2000, "o": 1500, "gu_down": 5000, "head": 9000}
    st = synthetic_timeline(L, ncta, work, release, skew)
    out = bench.phase_breakdown(st, L)
    for ph in bench.PHASES:
        # a phase ends at the LAST CTA's arrival: its work plus the arrival skew
        assert out[ph] == round(L * (work[ph] + (ncta - 1) * skew) / 1e3, 1), ph
    assert out["barriers"] == round(4 * L * release / 1e3, 1)
    assert out["lm_head"] == round(work["head"] / 1e3, 1)
    assert out["total"] == round(st[:, -1].max() / 1e3, 1)


def test_timeline_names_match_the_kernel_stamp_count():
    # 15 stamps per layer (13 for layer 0: no barrier before its q/k/v) + start + 4 for the head
    for L in (1, 2, 28):
        assert len(bench.timeline_names(L)) == 15 * L + 3


def test_phase_breakdown_rejects_a_wrong_stamp_count():
    st = np.zeros((2, 10), dtype=np.int64)
    assert "error" in bench.phase_breakdown(st, 2)
