"""Summaries of the per-instruction timestamps the kernel records in profile mode.

Create the handle with ``profile=1``; after a step, ``Megakernel.profile_records()``
returns int64 [n_sm, stride, 8] records (see ``mk_profile_read`` in include/mk.h).
This module turns them into the time breakdown of one step: per op, how long
SMs waited on counters, staged activations, computed, and when the last SM of
each (layer, op) finished -- the critical path through the layer chain.
"""

from __future__ import annotations

import argparse
import json
import sys

import numpy as np

OPS = {1: "qkv", 2: "attn", 3: "o", 4: "gu", 5: "down", 6: "lm"}


def flatten(rec: np.ndarray) -> list[dict]:
    rows = []
    n_sm, stride, _ = rec.shape
    for s in range(n_sm):
        for i in range(stride):
            r = rec[s, i]
            if r[1] == 0:
                continue
            rows.append(dict(sm=s, op=OPS.get(int(r[0]) & 0xFF, "?"), layer=int(r[0] >> 8) & 0xFFFF,
                             units=int(r[0] >> 24), t_start=int(r[1]), t_dep=int(r[2]),
                             t_done=int(r[3]), t_sig=int(r[4]), p_first=int(r[5]), p_last=int(r[6]),
                             c_wait=int(r[7]), c_pages=int(r[8]), p_wait=int(r[9]), p_pages=int(r[10])))
    return rows


def summarize(rec: np.ndarray) -> dict:
    """Aggregate one step's records (nanoseconds; 'critical' is the per-(layer, op)
    window from the first SM passing its wait to the last SM signalling)."""
    rows = flatten(rec)
    if not rows:
        return {}
    t0 = min(r["t_start"] for r in rows)
    t1 = max(r["t_sig"] for r in rows)
    per_op = {}
    for r in rows:
        d = per_op.setdefault(r["op"], dict(n=0, wait=0, work=0, signal=0, c_wait=0, c_pages=0,
                                            p_wait=0, p_pages=0))
        d["n"] += 1
        for k in ("c_wait", "c_pages", "p_wait", "p_pages"):
            d[k] += r[k]
        d["wait"] += r["t_dep"] - r["t_start"]
        d["work"] += r["t_done"] - r["t_dep"]
        d["signal"] += r["t_sig"] - r["t_done"]
    for d in per_op.values():
        for k in ("wait", "work", "signal"):
            d[k + "_us_mean"] = d[k] / d["n"] / 1e3
        d["c_wait_us_per_page"] = d["c_wait"] / max(1, d["c_pages"]) / 1e3
        d["p_wait_us_per_page"] = d["p_wait"] / max(1, d["p_pages"]) / 1e3
    phases = {}
    for r in rows:
        key = (r["layer"], r["op"])
        ph = phases.setdefault(key, dict(first_dep=r["t_dep"], last_sig=r["t_sig"], last_dep=r["t_dep"]))
        ph["first_dep"] = min(ph["first_dep"], r["t_dep"])
        ph["last_dep"] = max(ph["last_dep"], r["t_dep"])
        ph["last_sig"] = max(ph["last_sig"], r["t_sig"])
    crit = {}
    for (layer, op), ph in phases.items():
        c = crit.setdefault(op, [])
        c.append((ph["last_sig"] - ph["first_dep"]) / 1e3)
    return {
        "step_us": (t1 - t0) / 1e3,
        "per_op": {k: {kk: round(vv, 3) if isinstance(vv, float) else vv for kk, vv in v.items()}
                   for k, v in per_op.items()},
        "phase_us_mean": {op: round(float(np.mean(v)), 3) for op, v in crit.items()},
        "phase_end_us": sorted(((ph["last_sig"] - t0) / 1e3, layer, op)
                               for (layer, op), ph in phases.items()),
    }


def main(argv=None):
    """Profile one steady-state decode step of a workload and print its breakdown.

    python -m persistent_megakernel_02_b200.profile [--workload llama1b_bs1]
    """
    import os

    import torch

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from synth import configs

    from . import Megakernel

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama1b_bs1")
    ap.add_argument("--ring-pages", type=int, default=0)
    args = ap.parse_args(argv)
    wl = configs.WORKLOADS[args.workload]
    nb, P = wl["batch"], max(wl["prompt_lens"])
    cfg = configs.model_config(args.workload, max_seq=P + 8)
    w = synth.make_weights(cfg, device="cuda")
    mk = Megakernel(cfg, w, profile=1, ring_pages=args.ring_pages)
    prompts = [synth.prompt_tokens(cfg, b, wl["prompt_lens"][b]).tolist() for b in range(nb)]
    ids = torch.tensor([mk.prefill(b, prompts[b]) for b in range(nb)], dtype=torch.int32, device="cuda")
    pos = [len(p) for p in prompts]
    for t in range(2):
        mk.decode_step(ids, [p + t for p in pos], ids)
    mk.sync()
    mk.profile_records()  # resets the accumulators
    mk.decode_step(ids, [p + 2 for p in pos], ids)
    s = summarize(mk.profile_records())
    mk.close()
    out = {k: v for k, v in s.items() if k != "phase_end_us"}
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
