"""Summaries of the per-instruction timestamps the kernel records in profile mode.

Create the handle with ``profile=1``; after a step, ``Megakernel.profile_records()``
returns int64 [n_sm, stride, 32] records (see ``mk_profile_read`` in include/mk.h).
This module turns them into the time breakdown of one step: per op, how long
SMs waited on counters, staged activations, computed, and when the last SM of
each (layer, op) finished -- the critical path through the layer chain.
"""

from __future__ import annotations

import argparse
import json
import sys

import numpy as np

OPS = {1: "qkv", 2: "attn", 3: "o", 4: "gu", 5: "down", 6: "lm", 7: "gu_tc", 8: "lm_tc"}


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
                             c_wait=int(r[7]), c_pages=int(r[8]), p_wait=int(r[9]), p_pages=int(r[10]),
                             t_staged=int(r[11]), t_last_warp=int(r[12]), t_barrier=int(r[13]),
                             c_core=int(r[14]), c_epi=int(r[15]), slow_n=int(r[16]), slow_ns=int(r[17]),
                             t_stage_in=int(r[18]), t_stage_loaded=int(r[19]),
                             t_sum_x1=int(r[20]), t_sum_p=int(r[21]),
                             w_entry0=int(r[22]), w_entry1=int(r[23]), w_first1=int(r[24]), w_done0=int(r[25])))
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
                                            p_wait=0, p_pages=0, stage=0, units=0, tail=0, n_mv=0,
                                            bar=0, rel=0, c_core=0, c_epi=0, slow_n=0, slow_ns=0,
                                            st_call=0, st_load=0, st_rest=0, n_sum=0, sum_x1=0, sum_p=0,
                                            n_w=0, w_entry=0, w_entry_spread=0, w_first=0, w_done_first=0))
        d["n"] += 1
        if r["t_staged"] and r["t_last_warp"]:
            d["n_mv"] += 1
            d["stage"] += r["t_staged"] - r["t_dep"]          # activation load (+ RMSNorm)
            d["units"] += r["t_last_warp"] - r["t_staged"]    # pages, matvecs, epilogues
            d["tail"] += r["t_sig"] - r["t_last_warp"]        # CTA barrier + release
            d["bar"] += r["t_barrier"] - r["t_last_warp"]     # last warp -> barrier passed
            d["rel"] += r["t_sig"] - r["t_barrier"]           # the release itself
            if r["t_stage_in"] and r["t_stage_loaded"]:
                d["st_call"] += r["t_stage_in"] - r["t_dep"]          # into the staging function
                d["st_load"] += r["t_stage_loaded"] - r["t_stage_in"]  # activation loads back
                d["st_rest"] += r["t_staged"] - r["t_stage_loaded"]    # norm, shared-memory stores
            if r["w_entry0"] and r["w_first1"]:  # warp 0 of the consumers
                d["n_w"] += 1
                d["w_entry"] += r["w_entry0"] - r["t_staged"]          # staged -> warp 0 in its matvec
                d["w_first"] += r["w_first1"] - r["w_entry0"]          # -> its first page ready
            if r["t_sum_x1"] and r["t_stage_in"]:
                d["n_sum"] += 1
                d["sum_x1"] += r["t_sum_x1"] - r["t_stage_in"]     # residual x1 back
                d["sum_p"] += r["t_sum_p"] - r["t_sum_x1"]         # then the last partial
        for k in ("c_wait", "c_pages", "p_wait", "p_pages", "c_core", "c_epi", "slow_n", "slow_ns"):
            d[k] += r[k]
        d["wait"] += r["t_dep"] - r["t_start"]
        d["work"] += r["t_done"] - r["t_dep"]
        d["signal"] += r["t_sig"] - r["t_done"]
    for d in per_op.values():
        for k in ("wait", "work", "signal"):
            d[k + "_us_mean"] = d[k] / d["n"] / 1e3
        for k in ("stage", "units", "tail", "bar", "rel", "st_call", "st_load", "st_rest"):
            d[k + "_us_mean"] = d[k] / max(1, d["n_mv"]) / 1e3
        d["c_wait_us_per_page"] = d["c_wait"] / max(1, d["c_pages"]) / 1e3
        d["p_wait_us_per_page"] = d["p_wait"] / max(1, d["p_pages"]) / 1e3
        d["c_core_us_per_page"] = d["c_core"] / max(1, d["c_pages"]) / 1e3
        d["pages_per_instr_mean"] = d["c_pages"] / max(1, d["n_mv"])
        d["sum_x1_us_mean"] = d["sum_x1"] / max(1, d["n_sum"]) / 1e3
        for k in ("w_entry", "w_entry_spread", "w_first", "w_done_first"):
            d[k + "_us_mean"] = d[k] / max(1, d["n_w"]) / 1e3
        d["sum_p_us_mean"] = d["sum_p"] / max(1, d["n_sum"]) / 1e3
        d["slow_rereads_per_instr_mean"] = d["slow_n"] / d["n"]
        d["slow_us_per_reread"] = d["slow_ns"] / max(1, d["slow_n"]) / 1e3
        d["c_epi_us_per_page"] = d["c_epi"] / max(1, d["c_pages"]) / 1e3
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
    # the chain through a few middle layers: per op, when its first SM passed the
    # instruction barrier, when its last SM did, and when its last SM finished
    layers = sorted({layer for layer, _ in phases})
    mid = layers[len(layers) // 2 - 1: len(layers) // 2 + 1] if len(layers) > 2 else layers
    chain = []
    if mid:
        base = phases.get((mid[0], "qkv"), next(iter(phases.values())))["first_dep"]
        order = ["qkv", "attn", "o", "gu", "gu_tc", "down"]
        for layer in mid:
            for op in order:
                ph = phases.get((layer, op))
                if ph:
                    chain.append((layer, op, round((ph["first_dep"] - base) / 1e3, 2),
                                  round((ph["last_dep"] - base) / 1e3, 2), round((ph["last_sig"] - base) / 1e3, 2)))
    # spread between SMs in the streaming phases of the middle layer (and the LM
    # head): percentiles of each SM's start, units time and end, from the phase's
    # first start
    spread = {}
    for op in ("gu", "gu_tc", "down", "lm", "lm_tc"):
        lay = mid[0] if op not in ("lm", "lm_tc") and mid else None
        rs = [r for r in rows if r["op"] == op and (lay is None or r["layer"] == lay)]
        if not rs:
            continue
        f = min(r["t_dep"] for r in rs)
        q = lambda xs: [round(float(np.percentile(xs, k)) / 1e3, 2) for k in (0, 10, 50, 90, 100)]
        spread[op] = dict(dep=q([r["t_dep"] - f for r in rs]),
                          units=q([r["t_last_warp"] - r["t_staged"] for r in rs if r["t_staged"]]),
                          end=q([r["t_sig"] - f for r in rs]),
                          end_by_sm=[round((r["t_sig"] - f) / 1e3, 1) for r in sorted(rs, key=lambda r: r["sm"])])
    # Share of the SMs' time (n_sm x step) the consumers spent waiting on other SMs:
    # at instruction barriers (the slowest warp of the previous instruction, and the
    # hint-counter wait where enabled) and re-reading activations not yet written
    # (the polls that replace counter waits; summed over a CTA's 8 consumer warps,
    # so divided by 8), next to the share spent waiting for weight pages to land.
    n_sm = rec.shape[0]
    sm_time = n_sm * max(1, t1 - t0)
    barrier_ns = sum(r["t_dep"] - r["t_start"] for r in rows)
    poll_ns = sum(r["slow_ns"] for r in rows) / 8.0
    page_ns = sum(r["c_wait"] for r in rows) / 8.0
    wait_share = {"barrier": round(barrier_ns / sm_time, 4), "data_poll": round(poll_ns / sm_time, 4),
                  "barrier_plus_poll": round((barrier_ns + poll_ns) / sm_time, 4),
                  "page_wait": round(page_ns / sm_time, 4)}
    return {
        "step_us": (t1 - t0) / 1e3,
        "wait_share": wait_share,
        "spread_p0_10_50_90_100_us": spread,
        "chain_first_last_end_us": chain,
        "per_op": {k: {kk: round(vv, 3) if isinstance(vv, float) else vv for kk, vv in v.items()}
                   for k, v in per_op.items()},
        "phase_us_mean": {op: round(float(np.mean(v)), 3) for op, v in crit.items()},
        "phase_end_us": sorted(((ph["last_sig"] - t0) / 1e3, layer, op)
                               for (layer, op), ph in phases.items()),
    }


def markdown(s: dict, bench_us: float | None = None) -> str:
    """The summary of one profiled step as the tables of a text report: per-op
    means, the chain through the middle layers, the per-SM spread."""
    po, ph = s["per_op"], s["phase_us_mean"]
    out = []
    note = f" (bench without stamps: {bench_us:.1f} us)" if bench_us else ""
    out.append(f"Step in profile mode: {s['step_us']:.1f} us{note}.")
    out.append("")
    out.append("| op | window | barrier wait | stage | entry | first page | pages | dot/page | "
               "epilogue/page | page wait/page | slot wait/page | pages/SM |")
    out.append("|---|---|---|---|---|---|---|---|---|---|---|---|")
    for op in ("qkv", "attn", "o", "gu", "gu_tc", "down", "lm", "lm_tc"):
        if op not in po:
            continue
        d = po[op]
        if op == "attn":
            out.append(f"| attn | {ph.get('attn', 0):.2f} | {d['wait_us_mean']:.2f} | - | - | - | "
                       f"{d['work_us_mean']:.2f} (work) | - | - | - | - | - |")
            continue
        # tensor-core units record no per-page dot products (the MMAs run asynchronously)
        # and their pages' slot waits are not timed by the producer
        tc = op.endswith("_tc")
        core = "-" if tc else f"{d['c_core_us_per_page']:.2f}"
        slot = "-" if tc else f"{d['p_wait_us_per_page']:.2f}"
        out.append(f"| {op} | {ph.get(op, 0):.2f} | {d['wait_us_mean']:.2f} | {d['stage_us_mean']:.2f} | "
                   f"{d['w_entry_us_mean']:.2f} | {d['w_first_us_mean']:.2f} | {d['units_us_mean']:.2f} | "
                   f"{core} | {d['c_epi_us_per_page']:.2f} | "
                   f"{d['c_wait_us_per_page']:.2f} | {slot} | "
                   f"{d['pages_per_instr_mean']:.2f} |")
    out.append("")
    out.append("| layer | op | first start | last start | last end |")
    out.append("|---|---|---|---|---|")
    for layer, op, a, b, c in s["chain_first_last_end_us"]:
        out.append(f"| {layer} | {op} | {a} | {b} | {c} |")
    out.append("")
    sp = s["spread_p0_10_50_90_100_us"]
    out.append("Spread between SMs (percentiles 0/10/50/90/100 of each SM's end, from the phase's "
               "first start): " + "; ".join(f"{op} {sp[op]['end']}" for op in sp) + ".")
    ws = s.get("wait_share")
    if ws:
        out.append("")
        out.append(f"Wait share of the SMs' time (148 SMs x step): instruction barriers {100 * ws['barrier']:.1f} %, "
                   f"re-reads of activations not yet written {100 * ws['data_poll']:.1f} % "
                   f"(together {100 * ws['barrier_plus_poll']:.1f} %: the dependency waits that replace "
                   f"counter waits); waits for weight pages to land {100 * ws['page_wait']:.1f} %.")
    return "\n".join(out) + "\n"


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
    ap.add_argument("--markdown", action="store_true", help="print the report tables instead of JSON")
    ap.add_argument("--from-json", default=None, help="render a saved JSON summary (no GPU)")
    ap.add_argument("--ring-pages", type=int, default=0)
    ap.add_argument("--dyn-percent", type=int, default=0, help="claimed share of the streaming phases (0: none)")
    ap.add_argument("--tensor-core-units", type=int, default=0,
                    help="8-lane matvecs on tcgen05 (mk_options.tensor_core_units; 0 measured default)")
    ap.add_argument("--max-seq-extra", type=int, default=181,
                    help="max_seq = prompt + this (181: bench.py's default sizing, which sets the "
                         "attention slices per kv head)")
    args = ap.parse_args(argv)
    if args.from_json:
        with open(args.from_json) as f:
            saved = json.load(f)
        print(markdown(saved) if args.markdown else json.dumps(saved, indent=1))
        return
    wl = configs.WORKLOADS[args.workload]
    nb, P = wl["batch"], max(wl["prompt_lens"])
    cfg = configs.model_config(args.workload, max_seq=P + max(8, args.max_seq_extra))
    w = synth.make_weights(cfg, device="cuda")
    mk = Megakernel(cfg, w, profile=1, ring_pages=args.ring_pages, dyn_percent=args.dyn_percent,
                    tensor_core_units=args.tensor_core_units)
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
    print(markdown(out) if args.markdown else json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
