"""Llama-style dense decoder forward, written out from its definition (numpy).

TEST INFRASTRUCTURE ONLY -- never imported by the product path.

What is computed.  The Hazy Research megakernel article ("Stanford team's new
work lets Llama-1B reach millisecond inference", m.youleyou.com/wenzhang/2897217,
section "Megakernel: a deep-fusion design from scratch") names the fused
instructions of one decode step: RMSNorm + QKV projection + RoPE, attention, and
the MLP; the forum post "Two thousand four hundred kernel launches per token"
(zhichai.net/topic/178636135, reply) fixes the workload as Llama-3.2-1B at batch
1.  The layer itself is the standard Llama decoder layer, spelled out here:

    n  = x / sqrt(mean(x^2) + eps) * g_attn
    q, k, v = Wq n, Wk n, Wv n;  q, k rotated by RoPE at the token's position
    append (k, v) to the cache;  for each query head h with kv head g = h // (Hq/Hkv):
        o_h = softmax(q_h . K_g^T / sqrt(d)) V_g      over positions 0..pos
    x = x + Wo o
    n  = x / sqrt(mean(x^2) + eps) * g_mlp
    x = x + Wd (silu(Wg n) * (Wu n)),   silu(z) = z / (1 + e^-z)
    logits = W_lm (x / sqrt(mean(x^2) + eps) * g_final),  W_lm = embedding if tied
    greedy id = argmax(logits), lowest index on ties

Readings where the pages are silent (each listed in the design notes): RoPE
pairs are the half-split pairs (i, i + d/2); inverse frequencies theta^(-2i/d),
with the published Llama-3 frequency scaling when enabled; softmax scale
1/sqrt(d), no biases, no soft-capping; the current token attends to itself;
the KV cache is kept in the compute dtype (float32 by default).
"""

from __future__ import annotations

import math

import numpy as np


# --- building blocks ---------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return (x / np.sqrt(ms + x.dtype.type(eps))) * g


def rope_inv_freq(head_dim: int, theta: float, scaling: dict | None = None) -> np.ndarray:
    """Inverse frequencies theta^(-2i/d), i = 0..d/2-1, in float64.

    With ``scaling`` (keys factor, low_freq, high_freq, orig_max) the Llama-3
    rule is applied per frequency: wavelengths shorter than orig/high_freq are
    kept, longer than orig/low_freq are divided by ``factor``, and in between the
    two are blended linearly in orig/wavelength.
    """
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv = theta ** (-2.0 * i / head_dim)
    if not scaling:
        return inv
    factor = float(scaling["factor"])
    low, high = float(scaling["low_freq"]), float(scaling["high_freq"])
    orig = float(scaling["orig_max"])
    out = np.empty_like(inv)
    for j, f in enumerate(inv):
        wavelen = 2.0 * math.pi / f
        if wavelen < orig / high:
            out[j] = f
        elif wavelen > orig / low:
            out[j] = f / factor
        else:
            smooth = (orig / wavelen - low) / (high - low)
            out[j] = (1.0 - smooth) * f / factor + smooth * f
    return out


def rope_cos_sin(positions, inv_freq: np.ndarray, dtype=np.float32):
    """cos and sin of pos * inv_freq, computed in float64, shape [len(pos), d/2]."""
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(dtype), np.sin(ang).astype(dtype)


def rope_apply(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate half-split pairs (x[i], x[i + d/2]) by the angle whose cos/sin are given.

    x: [..., d]; cos, sin broadcastable to [..., d/2].
    """
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (z.dtype.type(1) + np.exp(-z))


def attention_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """One query position over a cache.

    q: [Hq, d]; K, V: [T, Hkv, d] (positions 0..T-1, all visible).
    Query head h reads kv head h // (Hq / Hkv).  Returns o: [Hq, d].
    """
    Hq, d = q.shape
    Hkv = K.shape[1]
    rep = Hq // Hkv
    scale = q.dtype.type(1.0 / math.sqrt(d))
    o = np.empty_like(q)
    for h in range(Hq):
        g = h // rep
        w = softmax((K[:, g, :] @ q[h]) * scale)
        o[h] = w @ V[:, g, :]
    return o


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Greedy id per row; np.argmax returns the first (lowest) index of the max."""
    return np.argmax(logits, axis=-1)


def top2_margin(logits: np.ndarray) -> np.ndarray:
    """Largest minus second-largest logit per row."""
    part = np.partition(logits, -2, axis=-1)
    return part[..., -1] - part[..., -2]


# --- weights -----------------------------------------------------------------

def _bf16_to_f32(t) -> np.ndarray:
    """Exact bf16 -> float32 upcast of a torch bf16 tensor (bits shifted left 16)."""
    import torch  # the oracle reads the shared seeded inputs, which are torch tensors

    u16 = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32)


def weights_to_numpy(w: dict) -> dict:
    """Convert the bf16 weight dict from :func:`synth.make_weights` to float32 numpy."""
    out = {}
    for k, v in w.items():
        if v is None:
            out[k] = None
        elif isinstance(v, list):
            out[k] = [_bf16_to_f32(t) for t in v]
        else:
            out[k] = _bf16_to_f32(v)
    return out


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), returned as float32.

    Diagnostic only: lets the oracle keep a bf16 KV cache like a GPU path that
    stores K and V in bf16, to separate that rounding from other differences.
    """
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16 << 16
    return bits.astype(np.uint32).view(np.float32)


# --- the model ---------------------------------------------------------------

class OracleModel:
    """fp32 (or fp64) forward of one decoder over float32 numpy weights."""

    def __init__(self, cfg: dict, weights: dict, dtype=np.float32, kv_round: str | None = None):
        self.cfg = cfg
        self.dt = np.dtype(dtype)
        # diagnostic only: store K, V rounded to "bf16" or "fp16" (default: compute dtype)
        self.kv_round = kv_round
        self.w = weights
        self.L = cfg["n_layers"]
        self.H = cfg["hidden"]
        self.Hq = cfg["n_heads"]
        self.Hkv = cfg["n_kv_heads"]
        self.d = cfg["head_dim"]
        self.eps = float(cfg["rms_eps"])
        scaling = None
        if cfg.get("rope_scaling", 0):
            scaling = dict(factor=cfg["rope_factor"], low_freq=cfg["rope_low_freq"],
                           high_freq=cfg["rope_high_freq"], orig_max=cfg["rope_orig_max"])
        self.inv_freq = rope_inv_freq(self.d, cfg["rope_theta"], scaling)

    def _m(self, name: str, layer: int | None = None) -> np.ndarray:
        a = self.w[name] if layer is None else self.w[name][layer]
        return a if a.dtype == self.dt else a.astype(self.dt)

    def _kv_rounded(self, a: np.ndarray) -> np.ndarray:
        if self.kv_round == "bf16":
            return round_to_bf16(a).astype(self.dt)
        return a.astype(np.float16).astype(self.dt)  # IEEE half, round to nearest even

    def _lm(self) -> np.ndarray:
        return self._m("embed") if self.cfg["tied"] else self._m("lm_head")

    # ---- token-by-token decode (the step the megakernel runs) ----

    def new_cache(self) -> dict:
        return {"K": [[] for _ in range(self.L)], "V": [[] for _ in range(self.L)]}

    def step(self, token: int, pos: int, cache: dict) -> np.ndarray:
        """Logits of one token at position ``pos``; appends its K/V to ``cache``.

        ``cache`` must already hold positions 0..pos-1.
        """
        Hq, Hkv, d = self.Hq, self.Hkv, self.d
        x = self._m("embed")[int(token)].copy()
        cos, sin = rope_cos_sin([pos], self.inv_freq, self.dt)
        for l in range(self.L):
            if len(cache["K"][l]) != pos:
                raise ValueError("cache does not hold positions 0..pos-1")
            n = rmsnorm(x, self._m("attn_norm", l), self.eps)
            q = (self._m("wq", l) @ n).reshape(Hq, d)
            k = (self._m("wk", l) @ n).reshape(Hkv, d)
            v = (self._m("wv", l) @ n).reshape(Hkv, d)
            q = rope_apply(q, cos[0], sin[0])
            k = rope_apply(k, cos[0], sin[0])
            if self.kv_round:
                k, v = self._kv_rounded(k), self._kv_rounded(v)
            cache["K"][l].append(k)
            cache["V"][l].append(v)
            o = attention_decode(q, np.stack(cache["K"][l]), np.stack(cache["V"][l]))
            x = x + self._m("wo", l) @ o.reshape(Hq * d)
            n = rmsnorm(x, self._m("mlp_norm", l), self.eps)
            a = silu(self._m("w_gate", l) @ n) * (self._m("w_up", l) @ n)
            x = x + self._m("w_down", l) @ a
        n = rmsnorm(x, self._m("final_norm"), self.eps)
        return self._lm() @ n

    def greedy(self, prompt, n_new: int):
        """Token-by-token greedy decode: returns (generated ids, logits per step).

        Step 0's logits are those of the last prompt position; step t >= 1 feeds
        generated id t-1 at position len(prompt) + t - 1.
        """
        cache = self.new_cache()
        logits = None
        for p, t in enumerate(prompt):
            logits = self.step(int(t), p, cache)
        ids, all_logits = [], []
        pos = len(prompt)
        for _ in range(n_new + 1):
            all_logits.append(logits)
            nxt = int(argmax_lowest(logits))
            ids.append(nxt)
            if len(ids) == n_new + 1:
                break
            logits = self.step(nxt, pos, cache)
            pos += 1
        return ids, all_logits

    # ---- whole sequence at once (causal), for long teacher-forced runs ----

    def forward_sequence(self, tokens, logits_at=None, q_chunk: int = 1024) -> np.ndarray:
        """Logits at positions ``logits_at`` (default: all) of a causal pass over
        ``tokens`` at positions 0..T-1.  Each query row is the definition above:
        its softmax runs over keys 0..its own position.  Query rows are processed
        in groups of ``q_chunk`` only to bound memory.
        """
        toks = np.asarray(tokens, dtype=np.int64)
        T = toks.shape[0]
        Hq, Hkv, d = self.Hq, self.Hkv, self.d
        rep = Hq // Hkv
        scale = self.dt.type(1.0 / math.sqrt(d))
        cos, sin = rope_cos_sin(np.arange(T), self.inv_freq, self.dt)
        X = self._m("embed")[toks].astype(self.dt)
        for l in range(self.L):
            n = rmsnorm(X, self._m("attn_norm", l), self.eps)
            Q = (n @ self._m("wq", l).T).reshape(T, Hq, d)
            K = (n @ self._m("wk", l).T).reshape(T, Hkv, d)
            V = (n @ self._m("wv", l).T).reshape(T, Hkv, d)
            Q = rope_apply(Q, cos[:, None, :], sin[:, None, :])
            K = rope_apply(K, cos[:, None, :], sin[:, None, :])
            if self.kv_round:
                K, V = self._kv_rounded(K), self._kv_rounded(V)
            O = np.empty((T, Hq, d), dtype=self.dt)
            for h in range(Hq):
                g = h // rep
                for i0 in range(0, T, q_chunk):
                    i1 = min(T, i0 + q_chunk)
                    S = (Q[i0:i1, h, :] @ K[:i1, g, :].T) * scale
                    # key j is visible to query i iff j <= i
                    mask = np.arange(i1)[None, :] > np.arange(i0, i1)[:, None]
                    S[mask] = -np.inf
                    O[i0:i1, h, :] = softmax(S, axis=-1) @ V[:i1, g, :]
            X = X + O.reshape(T, Hq * d) @ self._m("wo", l).T
            n = rmsnorm(X, self._m("mlp_norm", l), self.eps)
            A = silu(n @ self._m("w_gate", l).T) * (n @ self._m("w_up", l).T)
            X = X + A @ self._m("w_down", l).T
        sel = np.arange(T) if logits_at is None else np.asarray(logits_at, dtype=np.int64)
        n = rmsnorm(X[sel], self._m("final_norm"), self.eps)
        return n @ self._lm().T
