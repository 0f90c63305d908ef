"""Seeded synthetic inputs for the decode megakernel and for its oracle.

This module is the one place both sides share.  It holds none of the decoder's
arithmetic: only a counter-based integer hash that turns (seed, tensor id,
element index) into bf16 weights with an approximately normal N(0, sigma)
distribution, and into token ids.  Every step is integer arithmetic followed by
one IEEE float32 multiply and a round-to-nearest-even cast to bf16, so a CPU
and a GPU produce the same bits for the same arguments.

Hash: the "lowbias32" xorshift-multiply finalizer (constants 0x7feb352d and
0x846ca68b, published by C. Wellons in his integer-hash survey), applied twice
per draw.  Values are the centred sum of four 16-bit uniforms (Irwin-Hall,
n = 4), scaled to the requested standard deviation.

The five workload descriptions used by the tests and the benchmark live in
:mod:`synth.configs`.
"""

from __future__ import annotations

import math

import torch

MASK32 = 0xFFFFFFFF
_CHUNK = 1 << 25  # elements hashed per chunk (bounds the int64 temporaries)

# standard deviation of the sum of four independent uniforms on {0..65535}
_SUM4_STD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2**32 for int64 tensors holding values in [0, 2**32).

    The constant is split into 16-bit halves so no int64 product overflows.
    """
    lo = c & 0xFFFF
    hi = (c >> 16) & 0xFFFF
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & MASK32


def mix32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 finalizer on int64 tensors holding uint32 values."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _mix32_int(x: int) -> int:
    x &= MASK32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & MASK32
    x ^= x >> 15
    x = (x * 0x846CA68B) & MASK32
    x ^= x >> 16
    return x


def tensor_key(seed: int, tensor_id: int) -> int:
    """32-bit key of one tensor of one seed."""
    return _mix32_int(seed * 0x9E3779B9 + tensor_id * 0x85EBCA6B + 0x632BE5AB)


def _hash_pair(idx: torch.Tensor, key: int) -> tuple[torch.Tensor, torch.Tensor]:
    h1 = mix32(mix32(2 * idx) ^ key)
    h2 = mix32(mix32(2 * idx + 1) ^ key)
    return h1, h2


def normal_bf16(shape, seed: int, tensor_id: int, std: float = 0.02,
                device="cpu") -> torch.Tensor:
    """bf16 tensor of the given shape, ~N(0, std), bit-identical on any device."""
    n = 1
    for s in shape:
        n *= int(s)
    if n >= (1 << 31):
        raise ValueError("tensor too large for a 31-bit element counter")
    key = tensor_key(seed, tensor_id)
    scale = torch.tensor(std / _SUM4_STD, dtype=torch.float32, device=device)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for s0 in range(0, n, _CHUNK):
        s1 = min(n, s0 + _CHUNK)
        idx = torch.arange(s0, s1, dtype=torch.int64, device=device)
        h1, h2 = _hash_pair(idx, key)
        s = ((h1 & 0xFFFF) + (h1 >> 16) + (h2 & 0xFFFF) + (h2 >> 16)) - 131070
        # |s| <= 131070 < 2**24, so the int -> float32 conversion is exact; the one
        # multiply is IEEE round-to-nearest, the bf16 cast round-to-nearest-even.
        out[s0:s1] = (s.to(torch.float32) * scale).to(torch.bfloat16)
    return out.view(*shape)


def tokens(n: int, vocab: int, seed: int, tensor_id: int = 7001,
           device="cpu") -> torch.Tensor:
    """n token ids, uniform in [0, vocab), int32."""
    key = tensor_key(seed, tensor_id)
    idx = torch.arange(n, dtype=torch.int64, device=device)
    h = mix32(mix32(idx) ^ key)
    return ((h * vocab) >> 32).to(torch.int32)


# --- tensor ids of the decoder's weights (fixed so both sides agree) --------

EMBED_ID = 1
LM_HEAD_ID = 2
FINAL_NORM_ID = 3
_LAYER_BASE = 16
LAYER_NAMES = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")


def layer_tensor_id(layer: int, name: str) -> int:
    return _LAYER_BASE + 16 * layer + LAYER_NAMES.index(name)


def weight_shapes(cfg: dict) -> dict:
    """Row-major [out, in] shapes of every weight of one layer, and the globals."""
    H, d = cfg["hidden"], cfg["head_dim"]
    qd, kvd, F = cfg["n_heads"] * d, cfg["n_kv_heads"] * d, cfg["ffn"]
    return {
        "embed": (cfg["vocab"], H),
        "lm_head": (cfg["vocab"], H),
        "final_norm": (H,),
        "attn_norm": (H,),
        "wq": (qd, H),
        "wk": (kvd, H),
        "wv": (kvd, H),
        "wo": (H, qd),
        "mlp_norm": (H,),
        "w_gate": (F, H),
        "w_up": (F, H),
        "w_down": (H, F),
    }


def _gain(shape, seed, tid, cfg, device):
    jitter = cfg.get("norm_jitter", 0.0)
    if jitter == 0.0:
        return torch.ones(shape, dtype=torch.bfloat16, device=device)
    g = normal_bf16(shape, seed, tid, std=jitter, device=device).float() + 1.0
    return g.to(torch.bfloat16)


def make_weights(cfg: dict, device="cpu", seed: int | None = None,
                 zero_layers: bool = False) -> dict:
    """All decoder weights of ``cfg`` as bf16 tensors on ``device``.

    ``zero_layers`` zeroes every per-layer matrix (norm gains stay), which gives
    the closed-form special case used by the property tests.
    Returns a dict with 'embed', 'lm_head' (None when tied), 'final_norm' and one
    list per per-layer tensor name.
    """
    if seed is None:
        seed = cfg.get("weight_seed", 0)
    std = cfg.get("init_std", 0.02)
    shp = weight_shapes(cfg)
    w = {
        "embed": normal_bf16(shp["embed"], seed, EMBED_ID, std, device),
        "lm_head": None if cfg["tied"] else normal_bf16(shp["lm_head"], seed, LM_HEAD_ID, std, device),
        "final_norm": _gain(shp["final_norm"], seed, FINAL_NORM_ID, cfg, device),
    }
    for name in LAYER_NAMES:
        w[name] = []
    for layer in range(cfg["n_layers"]):
        for name in LAYER_NAMES:
            tid = layer_tensor_id(layer, name)
            if name.endswith("norm"):
                t = _gain(shp[name], seed, tid, cfg, device)
            elif zero_layers:
                t = torch.zeros(shp[name], dtype=torch.bfloat16, device=device)
            else:
                t = normal_bf16(shp[name], seed, tid, std, device)
            w[name].append(t)
    return w


def to_device(w: dict, device) -> dict:
    """The weight dict of :func:`make_weights` copied to ``device`` (bits unchanged).

    Generating on the CPU and copying keeps the device free of the generator's
    many small integer kernels (useful where a launch record is kept)."""
    out = {}
    for k, v in w.items():
        if v is None:
            out[k] = None
        elif isinstance(v, list):
            out[k] = [t.to(device) for t in v]
        else:
            out[k] = v.to(device)
    return out


def prompt_tokens(cfg: dict, seq: int, n: int, device="cpu") -> torch.Tensor:
    """Prompt of sequence ``seq``: n tokens uniform in [0, vocab), seed 1 + seq."""
    return tokens(n, cfg["vocab"], seed=cfg.get("prompt_seed", 1) + seq, device=device)


def teacher_tokens(cfg: dict, seq: int, n: int, device="cpu") -> torch.Tensor:
    """Seeded continuation tokens fed to both sides in teacher-forced parity runs."""
    return tokens(n, cfg["vocab"], seed=cfg.get("prompt_seed", 1) + seq, tensor_id=7002,
                  device=device)
