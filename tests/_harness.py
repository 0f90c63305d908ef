"""Shared helpers of the GPU parity tests (not collected as tests).

Runs the CUDA path through the C ABI (via the ctypes binding) and the CPU
oracle on the same seeded inputs, and compares them with the tolerances fixed
for this path: per step and sequence, logits max-abs <= 5e-2 and relative L2
<= 1e-2; greedy ids identical wherever the oracle's top-2 margin exceeds 0.1.
"""

from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import OracleModel, argmax_lowest, top2_margin, weights_to_numpy

MAX_ABS = 5e-2
REL_L2 = 1e-2
MARGIN = 0.1

# (case, worst max-abs, worst rel-L2, steps compared, ids compared) of every
# parity case that ran; tests/conftest.py prints them in the session summary
PARITY_RECORDS = []


def record(case, worst, steps, ids_checked):
    PARITY_RECORDS.append((case, float(worst[0]), float(worst[1]), int(steps), int(ids_checked)))


def gpu_weights(cfg, zero_layers=False):
    return synth.make_weights(cfg, device="cuda", zero_layers=zero_layers)


def oracle_for(cfg, w_gpu, dtype=np.float32):
    return OracleModel(cfg, weights_to_numpy(w_gpu), dtype)


def run_teacher_forced(mk, cfg, prompts, teacher, n_steps):
    """GPU: prefill each lane's prompt into its slot, then n_steps batched decode
    steps feeding teacher[b][t] at position len(prompt_b) + t.

    Returns (prefill_logits [nb][V], step_logits [n_steps][nb][V], step_ids [n_steps][nb]).
    """
    nb = len(prompts)
    V = cfg["vocab"]
    dev = torch.device("cuda")
    last = []
    for b, pr in enumerate(prompts):
        lg = torch.empty(V, dtype=torch.float32, device=dev)
        mk.prefill(b, [int(t) for t in pr], logits_last=lg)
        last.append(lg.cpu().numpy())
    logits = torch.empty((nb, V), dtype=torch.float32, device=dev)
    ids = torch.empty(nb, dtype=torch.int32, device=dev)
    tok = torch.empty(nb, dtype=torch.int32, device=dev)
    out_l, out_i = [], []
    for t in range(n_steps):
        tok.copy_(torch.tensor([int(teacher[b][t]) for b in range(nb)], dtype=torch.int32))
        pos = [len(prompts[b]) + t for b in range(nb)]
        mk.decode_step(tok, pos, ids, logits)
        mk.sync()
        out_l.append(logits.cpu().numpy().copy())
        out_i.append(ids.cpu().numpy().copy())
    return np.stack(last), np.stack(out_l), np.stack(out_i)


def oracle_teacher_forced(orc, prompt, teacher, n_steps):
    """Oracle logits at the last prompt position and at each teacher-forced step."""
    seq = np.concatenate([np.asarray(prompt), np.asarray(teacher[:n_steps])]).astype(np.int64)
    P = len(prompt)
    want = orc.forward_sequence(seq, logits_at=np.arange(P - 1, P + n_steps))
    return want[0], want[1:]


def compare_logits(got, want, what=""):
    """Assert the per-step tolerances; returns (max_abs, rel_l2)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU logits"
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= MAX_ABS, f"{what}: max-abs {err:.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return float(err), float(rel)


def compare_ids(got_id, want_logits, what=""):
    """Greedy ids must agree where the oracle's top-2 margin exceeds MARGIN;
    elsewhere the GPU id must be one of the oracle's near-ties."""
    want_logits = np.asarray(want_logits)
    wid = int(argmax_lowest(want_logits))
    margin = float(top2_margin(want_logits))
    if margin > MARGIN:
        assert int(got_id) == wid, f"{what}: id {got_id} != oracle {wid} (margin {margin:.3f})"
        return True
    assert want_logits[int(got_id)] >= want_logits[wid] - MARGIN - MAX_ABS, \
        f"{what}: id {got_id} is not a near-tie of the oracle's {wid}"
    return False
