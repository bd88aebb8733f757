"""Summaries of the library's device timeline trace (ocrdec_set_trace /
ocrdec_read_trace).

Every traced CTA contributes (start, duration, kernel tag, SM).  A launch is
the cluster of records of one tag that overlap in time (launches of one tag
never overlap each other within a step).  The summary gives, per tag, the
number of launches and their mean span (first CTA start to last CTA end), and
the idle time of the whole window: time covered by no CTA at all.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np

TAGS = {1: "qkv", 6: "dense_gate_up", 7: "dense_down", 8: "lm_head_verify+accept", 9: "lm_head_draft",
        10: "draft_fc", 11: "moe_ffn (routing+experts+combine)", 40: "norm+qkv+rope+attention+o_proj(+router partials)",
        41: "attention (cluster rank 0)", 42: "verify_setup", 43: "draft_setup"}


def launches(rec: np.ndarray) -> List[dict]:
    """Group records into launches: per tag, sort by start and cut where a record
    starts after every earlier record of the group has ended."""
    out = []
    for tag in np.unique(rec["tag"]):
        r = rec[rec["tag"] == tag]
        t0 = r["t0"].astype(np.int64)
        t1 = t0 + r["dt"].astype(np.int64)
        order = np.argsort(t0)
        t0, t1 = t0[order], t1[order]
        start, end, n = t0[0], t1[0], 1
        for a, b in zip(t0[1:], t1[1:]):
            if a > end:
                out.append(dict(tag=int(tag), t0=int(start), t1=int(end), ctas=n))
                start, end, n = a, b, 1
            else:
                end = max(end, b)
                n += 1
        out.append(dict(tag=int(tag), t0=int(start), t1=int(end), ctas=n))
    out.sort(key=lambda d: d["t0"])
    return out


def summary(rec: np.ndarray, steps: int) -> Dict:
    if len(rec) == 0:
        return {}
    L = launches(rec)
    t_begin = min(d["t0"] for d in L)
    t_end = max(d["t1"] for d in L)
    # busy = union of launch spans
    busy, cur0, cur1 = 0, None, None
    for d in L:
        if cur0 is None:
            cur0, cur1 = d["t0"], d["t1"]
        elif d["t0"] > cur1:
            busy += cur1 - cur0
            cur0, cur1 = d["t0"], d["t1"]
        else:
            cur1 = max(cur1, d["t1"])
    busy += cur1 - cur0
    per_tag = {}
    for d in L:
        name = TAGS.get(d["tag"], str(d["tag"]))
        e = per_tag.setdefault(name, {"launches": 0, "span_us": 0.0})
        e["launches"] += 1
        e["span_us"] += (d["t1"] - d["t0"]) / 1e3
    for tag in np.unique(rec["tag"]):
        r = rec[rec["tag"] == tag]
        e = per_tag[TAGS.get(int(tag), str(int(tag)))]
        # mean per-CTA phase ends (us after the CTA's dependency wait)
        e["cta_phase_us"] = [round(float(np.mean(r[f])) / 1e3, 2) for f in ("d1", "d2", "dt")]
        e["cta_phase_max_us"] = [round(float(np.max(r[f])) / 1e3, 2) for f in ("d1", "d2", "dt")]
        e["ctas_per_launch"] = round(len(r) / e["launches"], 1)
    for e in per_tag.values():
        e["mean_us"] = e["span_us"] / e["launches"]
        e["per_step_us"] = e["span_us"] / steps
    return {"steps": steps, "window_us": (t_end - t_begin) / 1e3, "per_step_us": (t_end - t_begin) / 1e3 / steps,
            "idle_us_per_step": ((t_end - t_begin) - busy) / 1e3 / steps, "launches_per_step": len(L) / steps,
            "per_tag": dict(sorted(per_tag.items(), key=lambda kv: -kv[1]["span_us"]))}


def format_summary(s: Dict) -> str:
    lines = [f"window {s['window_us']:.1f} us over {s['steps']} steps: {s['per_step_us']:.1f} us/step, "
             f"idle {s['idle_us_per_step']:.1f} us/step, {s['launches_per_step']:.1f} launches/step"]
    for name, e in s["per_tag"].items():
        lines.append(f"  {name:24s} {e['launches']:5d} launches  mean {e['mean_us']:8.2f} us  "
                     f"{e['per_step_us']:8.1f} us/step  ctas {e.get('ctas_per_launch')}  "
                     f"cta phases {e.get('cta_phase_us')} max {e.get('cta_phase_max_us')}")
    return "\n".join(lines)
