"""The decoder shapes and decode workloads exercised by the tests and the benchmark.

Each workload names a model shape (fields match ``mk_config`` in include/mk.h)
plus the batch, prompt lengths and number of greedy decode steps.  Weights are
seeded random-init bf16 ~N(0, 0.02) from :mod:`synth`, norm gains 1.0.

RoPE: inverse frequencies theta**(-2i/d) over half-split pairs (i, i + d/2);
"llama3" scaling uses the published Llama-3.2 parameters (factor 32, low-frequency
factor 1, high-frequency factor 4, original context 8192).
"""

from __future__ import annotations

import copy

_LLAMA3_SCALING = dict(rope_scaling=1, rope_factor=32.0, rope_low_freq=1.0,
                       rope_high_freq=4.0, rope_orig_max=8192)
_NO_SCALING = dict(rope_scaling=0, rope_factor=1.0, rope_low_freq=1.0,
                   rope_high_freq=1.0, rope_orig_max=0)

TINY = dict(n_layers=2, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=1024,
            vocab=4096, tied=1, rms_eps=1e-5, rope_theta=500000.0, kv_dtype=0, **_NO_SCALING)

LLAMA_1B = dict(n_layers=16, hidden=2048, n_heads=32, n_kv_heads=8, head_dim=64, ffn=8192,
                vocab=128256, tied=1, rms_eps=1e-5, rope_theta=500000.0, kv_dtype=0,
                **_LLAMA3_SCALING)

# The 8B workload states no KV-cache type; bf16 K/V rounding alone moves its
# 32-layer logits past the parity tolerance against the fp32 oracle, so its
# cache is fp16 (same bytes, 3 more mantissa bits).  kv_dtype: 0 bf16, 1 fp16.
LLAMA_8B = dict(n_layers=32, hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128, ffn=14336,
                vocab=128256, tied=0, rms_eps=1e-5, rope_theta=500000.0, kv_dtype=1, **_NO_SCALING)


def _wl(name, model, batch, prompt_lens, decode_steps, desc):
    return dict(name=name, model=model, batch=batch, prompt_lens=list(prompt_lens),
                decode_steps=decode_steps, desc=desc)


WORKLOADS = {
    "tiny": _wl("tiny", TINY, 1, [8], 16,
                "tiny Llama-style decoder, 2 layers, hidden 256, bs1, 8 prompt -> 16 greedy"),
    "llama1b_bs1": _wl("llama1b_bs1", LLAMA_1B, 1, [32], 128,
                       "Llama-3.2-1B shape, bs1, 32 prompt -> 128 greedy"),
    "llama1b_long": _wl("llama1b_long", LLAMA_1B, 1, [8192], 64,
                        "Llama-3.2-1B shape, bs1, 8192-token KV prefill -> 64 decode steps"),
    "llama1b_bs4": _wl("llama1b_bs4", LLAMA_1B, 4, [512 + 128 * i for i in range(4)], 128,
                       "Llama-3.2-1B shape, batch 4, prompts 512/640/768/896 -> 128 decode steps"),
    "llama1b_bs8": _wl("llama1b_bs8", LLAMA_1B, 8, [512 + 128 * i for i in range(8)], 128,
                       "Llama-3.2-1B shape, batch 8, prompts 512..1408 -> 128 decode steps"),
    "llama8b_bs1": _wl("llama8b_bs1", LLAMA_8B, 1, [2048], 128,
                       "Llama-3-8B shape, untied, bs1, 2048 prompt -> 128 greedy"),
}


def model_config(workload: str | dict, max_batch: int | None = None,
                 max_seq: int | None = None, **overrides) -> dict:
    """mk_config fields for a workload (a copy; overrides applied last)."""
    wl = WORKLOADS[workload] if isinstance(workload, str) else workload
    cfg = copy.deepcopy(wl["model"])
    cfg["max_batch"] = max_batch if max_batch is not None else wl["batch"]
    cfg["max_seq"] = max_seq if max_seq is not None else max(wl["prompt_lens"]) + wl["decode_steps"]
    cfg.update(overrides)
    return cfg


def weight_bytes(cfg: dict) -> int:
    """Bytes of every weight one decode step streams (bf16)."""
    H, d, F, V, L = cfg["hidden"], cfg["head_dim"], cfg["ffn"], cfg["vocab"], cfg["n_layers"]
    qd, kvd = cfg["n_heads"] * d, cfg["n_kv_heads"] * d
    per_layer = (qd + 2 * kvd) * H + H * qd + 3 * F * H + 2 * H
    return 2 * (L * per_layer + V * H + H)


def kv_bytes_per_pos(cfg: dict) -> int:
    """bf16 K and V bytes of one position over all layers."""
    return 2 * 2 * cfg["n_layers"] * cfg["n_kv_heads"] * cfg["head_dim"]


def step_bytes(cfg: dict, positions) -> int:
    """Algorithmic HBM bytes of one decode step at the given per-lane positions:
    every weight once, one embedding row per lane, the KV cache of positions
    0..pos read per lane (pos + 1 positions), and the K/V of the new position
    written per lane."""
    kvp = kv_bytes_per_pos(cfg)
    emb = 2 * cfg["hidden"]
    return weight_bytes(cfg) + sum(emb + (int(p) + 2) * kvp for p in positions)
