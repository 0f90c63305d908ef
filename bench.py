"""Decode-step benchmark of the persistent megakernel on B200.

One "step" is one decode step of the whole model (every layer plus the LM head
and greedy argmax) for the workload's batch, i.e. one launch of the persistent
kernel.  Default workload: the Llama-3.2-1B shape at batch 1 (32-token prompt,
then greedy decode, tokens chained on the device), seeded random-init bf16
weights.  The weights (2.47 GB) are far larger than L2 (126 MB), so no L2 flush
is needed between steps.

Prints ONE JSON line on rank 0.  Runs as N independent replicas under torchrun
(one process per GPU); the path does not shard, so there is no collective on the
data path -- only a barrier and a max-over-ranks of the device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mk|reference]
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/decode step (bs1, Llama-3.2-1B shape); achieved HBM TB/s vs ~8 TB/s roofline"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # nvidia-smi takes a while to start: begin timing once it samples
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.lines.clear()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            t0 = time.time()  # a short timed region: wait for at least two samples
            while len(self.lines) < 2 and time.time() - t0 < 0.5:
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


KERNEL_SOURCES = ["mk_kernel.cuh", "mk_device.cuh", "mk_matvec.cuh", "mk_tc.cuh", "mk_plan.h", "mk_sched.cpp", "mk_api.cu"]


def kernel_src_hash() -> str:
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "persistent_megakernel_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per decode step from the committed ncu summary (a capture of one
    single-step launch of the kernel), if it was taken on this workload with the
    current kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", f"mk_decode_kernel_{workload}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_src_sha256_16") != kernel_src_hash():
        return None
    return float(kv["dram_bytes_per_step"])


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest value any rank reports (device time of the slowest replica).
    ``dist`` is torch.distributed with an initialised group, or None for one rank."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(cfg, prompt, n_steps, w_host=None, time_budget_s=25.0, warmup=0):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload:
    the prompt and `warmup` greedy decode steps run untimed, then up to n_steps
    greedy decode steps are timed (stopping once the budget is spent).  Returns
    (us per step, timed steps, threads)."""
    import numpy as np

    from oracle import OracleModel, argmax_lowest

    orc = OracleModel(cfg, w_host, np.float32)
    cache = orc.new_cache()
    logits = None
    for p, t in enumerate(prompt):
        logits = orc.step(int(t), p, cache)
    pos = len(prompt)
    tok = int(argmax_lowest(logits))
    for _ in range(warmup):
        logits = orc.step(tok, pos, cache)
        tok = int(argmax_lowest(logits))
        pos += 1
    t0 = time.perf_counter()
    done = 0
    while done < n_steps:
        logits = orc.step(tok, pos, cache)
        tok = int(argmax_lowest(logits))
        pos += 1
        done += 1
        if time.perf_counter() - t0 > time_budget_s:
            break
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OPENBLAS_NUM_THREADS", os.cpu_count() or 1))
    return 1e6 * dt / done, done, threads


def host_weights(w):
    from oracle import weights_to_numpy

    return weights_to_numpy(w)


def run_reference(args, cfg, wl):
    """--impl reference: the oracle on the host cores, same metric and config."""
    import torch  # noqa: F401  (seeded inputs are torch tensors)

    import synth

    w = synth.make_weights(cfg, device="cpu")
    prompt = synth.prompt_tokens(cfg, 0, wl["prompt_lens"][0]).numpy()
    us, done, threads = oracle_sample(cfg, prompt, max(1, args.steps), host_weights(w),
                                      time_budget_s=args.ref_budget, warmup=args.warmup)
    sample = (f"{done} greedy decode steps timed after an untimed {len(prompt)}-token prompt and "
              f"{args.warmup} untimed steps, workload {wl['name']}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us/step",
        "n_gpus": args.gpus, "steps": done, "warmup": args.warmup, "ms_per_step": round(us / 1000, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": _config_obj(wl, cfg),
        "cpu_baseline": {"value": round(us, 1), "unit": "us/step", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(us, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config_obj(wl, cfg):
    return {"workload": wl["name"], "desc": wl["desc"], "batch": wl["batch"],
            "prompt_lens": wl["prompt_lens"], "layers": cfg["n_layers"], "hidden": cfg["hidden"],
            "vocab": cfg["vocab"], "parallelism": "replicas", "l2": "weights 2.47 GB >> 126 MB L2; no flush"
            if cfg["hidden"] >= 2048 else "small model, L2-resident"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama1b_bs1")
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=25.0)
    ap.add_argument("--region-cut", type=int, default=0, choices=[0, 1],
                    help="1: each decode step is two launches (decoder layers, then LM head)")
    ap.add_argument("--tensor-core-units", type=int, default=0, choices=[0, 1, 2, 3, 4],
                    help="8-lane matvecs on tcgen05: 0 measured default, 1 none, 2 LM head, 3 gate/up, 4 both")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per decode step from an ncu capture of this kernel (optional)")
    args = ap.parse_args()
    from synth import configs

    wl = configs.WORKLOADS[args.workload]
    ws, rank, local = _dist()
    nb = wl["batch"]
    P = max(wl["prompt_lens"])
    e2e_steps = min(args.steps, 32)
    max_seq = P + args.warmup + args.steps + 8 + e2e_steps + 8
    cfg = configs.model_config(args.workload, max_seq=max_seq)

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg, wl)
        return

    import torch

    import synth
    from persistent_megakernel_02_b200 import Megakernel

    torch.cuda.set_device(local)
    pg = None
    if ws > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    w = synth.make_weights(cfg, device="cuda")
    mk = Megakernel(cfg, w, device=local, region_cut=args.region_cut, tensor_core_units=args.tensor_core_units)
    stream = torch.cuda.current_stream()
    prompts = [synth.prompt_tokens(cfg, b, wl["prompt_lens"][b]).tolist() for b in range(nb)]
    firsts = [mk.prefill(b, prompts[b]) for b in range(nb)]
    # prefill time of the workload's prompts (again, warm: the same rows are rewritten)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for b in range(nb):
        mk.prefill(b, prompts[b], want_id=False, stream=stream)
    p1.record(stream)
    torch.cuda.synchronize()
    prefill_ms = p0.elapsed_time(p1)
    ids = torch.tensor(firsts, dtype=torch.int32, device="cuda")
    pos0 = [len(p) for p in prompts]

    out = torch.empty((max(args.steps, args.warmup), nb), dtype=torch.int32, device="cuda")

    def steps(t0, n):
        """n chained decode steps in one launch, starting at step t0 (ids fed back)."""
        mk.decode_steps(ids, [p + t0 for p in pos0], n, out, stream=stream)
        ids.copy_(out[n - 1])

    steps(0, args.warmup)
    mk.sync(stream)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        steps(args.warmup, args.steps)
        ev1.record(stream)
        torch.cuda.synchronize()
    mk.sync(stream)
    ms = max_over_ranks(ev0.elapsed_time(ev1), pg, "cuda")
    if pg:
        pg.barrier()
    us_step = 1000.0 * ms / args.steps
    # algorithmic bytes of the timed steps (weights + KV read/write at each step's positions)
    total_bytes = sum(configs.step_bytes(cfg, [p + t for p in pos0])
                      for t in range(args.warmup, args.warmup + args.steps))
    bytes_step = total_bytes / args.steps
    gbs = total_bytes / (ms * 1e-3) / 1e9

    # the same steps launched one at a time (for comparison; not the headline)
    base1 = args.warmup + args.steps
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(8):
        mk.decode_step(ids, [p + base1 + t for p in pos0], ids, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    us_single = 1000.0 * e0.elapsed_time(e1) / 8

    # end to end through the C ABI with host buffers (H2D tokens, D2H ids per step)
    base = args.warmup + args.steps + 8
    mk_ids = list(firsts)
    t0 = time.perf_counter()
    for t in range(e2e_steps):
        mk_ids, _ = mk.decode_step_host(mk_ids, [p + base + t for p in pos0])
    e2e_us = 1e6 * (time.perf_counter() - t0) / e2e_steps
    mk.close()
    e2e_us = max_over_ranks(e2e_us, pg, "cuda")

    peak, peak_kind = _peaks()
    line = {
        "metric": METRIC, "value": round(us_step, 2), "unit": "us/step", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us_step / 1000, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init bf16 weights, seeded prompt, greedy ids chained on device)",
        "config": _config_obj(wl, cfg),
        "hbm_tbs": round(gbs / 1000, 3),
        "frac_of_8tbs": round(gbs / 8000, 3),
        "bytes_per_step": int(bytes_step),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                     "traffic": args.traffic_bytes if args.traffic_bytes is not None
                     else recorded_traffic(args.workload),
                     "kernel": "mk::mk_decode_kernel<1>" if nb == 1 else f"mk::mk_decode_kernel<{nb}>"},
        "e2e": {"value": round(e2e_us, 2), "unit": "us/step", "h2d_bytes_per_step": 4 * nb,
                "d2h_bytes_per_step": 4 * nb},
        "gpu_launches": 2 * args.steps if args.region_cut else 1,
        "prefill": {"tokens": sum(len(p) for p in prompts), "ms": round(prefill_ms, 3),
                    "tokens_per_s": round(sum(len(p) for p in prompts) / (prefill_ms * 1e-3), 1),
                    "path": "batched (tcgen05 GEMMs + causal attention), last token through the decode kernel"
                    if min(len(p) for p in prompts) >= 17 else "token by token through the decode kernel"},
        "region_cut": args.region_cut,
        "tensor_core_units": args.tensor_core_units,
        "us_per_step_one_launch_per_step": round(us_single, 2),
        "clocks": clk.summary(),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        wh = host_weights(w)
        us, done, threads = oracle_sample(cfg, prompts[0], 64, wh)
        line["cpu_baseline"] = {"value": round(us, 1), "unit": "us/step", "cores": threads,
                                "kind": "oracle",
                                "sample": f"{done} greedy decode steps of lane 0 after an untimed "
                                          f"{len(prompts[0])}-token prompt (numpy fp32, OpenBLAS)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
