"""Decode the megakernel's per-task trace (MK_DEBUG_TRACE).

Per CTA the trace holds records of 16 uint32.  Record 0 is a header
``{records, notifier batches, notified tasks, fence ns}``; records 1.. are
tasks ``{family, index, t_pop, t_ready, t_go, t_done, t_notified, t_cstart,
t_cend, t_issue, t_data, ...}``, times being the low 32 bits of the global
timer in ns.  ``t_issue``: the producer issued the task's copies; ``t_pop``:
the controller took it; ``t_ready``: its event had fired; ``t_go``: it was
released; ``t_cstart``/``t_cend``: the compute warps started / finished it;
``t_data``: its first ring slot was full; ``t_done``: the controller saw it
finish; ``t_notified``: its event counter was decremented.  GEMV tasks also
record ``t_staged`` (activation staged), ``t_math`` (compute warp 0's
products done), ``t_red`` (partial tiles summed, epilogue starts),
``t_epi`` (compute warp 0's epilogue items written) and ``t_loads`` (the
staging's first rows loaded).
"""
from __future__ import annotations

import json

FIELDS = ["family", "index", "pop", "ready", "go", "done", "notified", "cstart", "cend", "issue", "data",
          "staged", "math", "red", "epi", "loads"]


def records(trace, fam_names):
    """List of dicts, one per task, from a ``[n_sm][cap][16]`` int32 tensor.

    Times are unwrapped against the CTA's first ``pop`` and returned in ns.
    """
    t = trace.cpu().to(dtype=__import__("torch").int64) & 0xFFFFFFFF
    out = []
    base = None
    for sm in range(t.shape[0]):
        n = int(t[sm, 0, 0])
        rows = t[sm, 1:min(n, t.shape[1] - 1) + 1].tolist()
        if not rows:
            continue
        if base is None:
            base = rows[0][2]
        for v in rows:
            rec = {"sm": sm}
            fam = v[0]
            rec["family"] = fam_names[fam] if 0 <= fam < len(fam_names) else str(fam)
            rec["index"] = v[1]
            for i, k in enumerate(FIELDS[2:], start=2):
                rec[k] = ((v[i] - base + (1 << 31)) % (1 << 32)) - (1 << 31) if v[i] else None
            out.append(rec)
    return out


def header(trace):
    t = trace.cpu().to(dtype=__import__("torch").int64) & 0xFFFFFFFF
    return [{"records": int(r[0]), "batches": int(r[1]), "notified": int(r[2]), "fence_ns": int(r[3])}
            for r in t[:, 0].tolist()]


def summary(recs):
    """Per-op totals: task count, mean compute time, mean wait for the event,
    mean notify latency (us)."""
    if not recs:
        return {}
    recs = [r for r in recs if r["go"] is not None]
    t0 = min(r["pop"] for r in recs)
    t1 = max(max(r["done"] or 0, r["notified"] or 0) for r in recs)
    by = {}
    for r in recs:
        op = r["family"].split(".")[0]
        d = by.setdefault(op, {"tasks": 0, "compute_us": 0.0, "wait_us": 0.0, "notify_us": 0.0,
                               "gap_us": 0.0})
        d["tasks"] += 1
        if r["cend"] is not None and r["cstart"] is not None:
            d["compute_us"] += (r["cend"] - r["cstart"]) / 1e3
        d["wait_us"] += max(0, r["ready"] - r["pop"]) / 1e3
        d["gap_us"] += max(0, r["go"] - r["ready"]) / 1e3
        if r["notified"] is not None and r["done"] is not None:
            d["notify_us"] += (r["notified"] - r["done"]) / 1e3
    for d in by.values():
        n = d["tasks"]
        for k in ("compute_us", "wait_us", "notify_us", "gap_us"):
            d[k] = round(d[k] / n, 3)
    return {"span_us": (t1 - t0) / 1e3, "ops": by}


def chrome_trace(recs, path):
    """Write a Chrome trace (chrome://tracing) with one row per SM."""
    if not recs:
        return
    ev = []
    for r in recs:
        if r["cstart"] is not None and r["cend"] is not None and r["cend"] > r["cstart"]:
            ev.append({"name": r["family"], "ph": "X", "pid": 0, "tid": r["sm"], "ts": r["cstart"] / 1e3,
                       "dur": (r["cend"] - r["cstart"]) / 1e3, "args": {"index": r["index"]}})
        if r["ready"] > r["pop"]:
            ev.append({"name": "wait", "ph": "X", "pid": 1, "tid": r["sm"], "ts": r["pop"] / 1e3,
                       "dur": (r["ready"] - r["pop"]) / 1e3})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev}, f)
