"""bench.py's reduction of the step kernel's timeline stamps to per-phase critical-path times
(CPU only): a synthetic 3-CTA, 2-layer timeline with known phase and barrier durations."""

import numpy as np

import bench


def synthetic_timeline(L, ncta, work_ns, release_ns, skew_ns):
    """Stamps in the kernel's order: start, [staged], then per phase arrive/exit(/staged) ... ,
    head arrive/exit/staged, end.  CTA c arrives c * skew_ns after CTA 0 at every barrier; every
    CTA leaves a barrier release_ns after the last arrival and stages its input in 0 ns."""
    rows = [[] for _ in range(ncta)]
    t = 0
    for r in rows:
        r += [t, t]  # start, L0.qkv.staged
    order = ["qkv", "attn", "o", "gu", "down"]
    for l in range(L):
        for j, ph in enumerate(order):
            if l == 0 and j == 0:
                continue
            prev = order[j - 1] if j > 0 else "down"
            t += work_ns[prev]
            last = t + (ncta - 1) * skew_ns
            for c, r in enumerate(rows):
                r.append(t + c * skew_ns)  # arrive
            t = last + release_ns
            for r in rows:
                r.append(t)  # exit
                if ph != "attn":
                    r.append(t)  # staged
    t += work_ns["down"]
    last = t + (ncta - 1) * skew_ns
    for c, r in enumerate(rows):
        r.append(t + c * skew_ns)
    t = last + release_ns
    for r in rows:
        r += [t, t]  # head exit, staged
    t += work_ns["head"]
    for r in rows:
        r.append(t)  # end
    return np.array(rows, dtype=np.int64)


def test_phase_breakdown_recovers_known_durations():
    L, ncta, release, skew = 2, 3, 700, 40
    work = {"qkv": 1000, "attn": 2000, "o": 1500, "gu": 5000, "down": 3000, "head": 9000}
    st = synthetic_timeline(L, ncta, work, release, skew)
    out = bench.phase_breakdown(st, L)
    for ph in ("qkv", "attn", "o", "gu", "down"):
        # a phase ends at the LAST CTA's arrival: its work plus the arrival skew
        assert out[ph] == round(L * (work[ph] + (ncta - 1) * skew) / 1e3, 1), ph
    assert out["barriers"] == round(5 * L * release / 1e3, 1)
    assert out["lm_head"] == round(work["head"] / 1e3, 1)
    assert out["total"] == round(st[:, -1].max() / 1e3, 1)


def test_phase_breakdown_rejects_a_wrong_stamp_count():
    st = np.zeros((2, 10), dtype=np.int64)
    assert "error" in bench.phase_breakdown(st, 2)
