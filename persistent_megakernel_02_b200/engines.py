"""Which engine should a decode step's matvecs run on?  Times mk_matvec_engine
(CUDA cores vs tcgen05 tensor cores) on the streaming batched matvec of the
decoder's shapes, per batch size, against the measured HBM copy bandwidth.

  python -m persistent_megakernel_02_b200.engines [--reps 10]

Prints one JSON object: per (shape, nb, engine) the mean time of one pass over
the weight matrix (CUDA events on the launching stream, after warm-up; the
matrices are larger than L2, so no flush is needed) and the achieved GB/s of
the weight stream.
"""

from __future__ import annotations

import argparse
import json
import os

SHAPES = {
    # name: (rows, K) -- bf16 weight matrices of the Llama-3.2-1B decoder
    "gate_up_1b": (16384, 2048),   # W_gate and W_up stacked: 64 MiB
    "lm_head_1b": (128256, 2048),  # tied embedding / LM head: 501 MiB
}


def _peak_gbs():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = os.path.join(root, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def main(argv=None):
    import torch

    from . import matvec_engine, matvec_engine_status

    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args(argv)
    peak, kind = _peak_gbs()
    out = {"peak_gbs": peak, "peak_kind": kind, "runs": []}
    for name, (rows, K) in SHAPES.items():
        g = torch.Generator(device="cpu").manual_seed(rows)
        W = (torch.randn(rows, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
        for nb in (1, 2, 4, 8):
            X = torch.randn(nb, K, generator=g).float().cuda()
            ref = None
            for engine in ("cuda_cores", "tcgen05"):
                Y = torch.empty((nb, rows), device="cuda")
                for _ in range(args.warmup):
                    matvec_engine(engine, W, X, Y)
                matvec_engine_status()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(args.reps):
                    matvec_engine(engine, W, X, Y)
                e1.record()
                matvec_engine_status()
                us = 1000.0 * e0.elapsed_time(e1) / args.reps
                if ref is None:
                    ref = (X.double() @ W.double().t())
                rel = ((Y.double() - ref).norm() / ref.norm()).item()
                gbs = rows * K * 2 / (us * 1e-6) / 1e9
                out["runs"].append({"shape": name, "rows": rows, "K": K, "nb": nb, "engine": engine,
                                    "us": round(us, 2), "weight_gbs": round(gbs, 1),
                                    "frac_of_peak": round(gbs / peak, 4), "rel_l2_vs_fp64": rel})
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
