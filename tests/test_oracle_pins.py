"""Pins of the CPU oracle to facts other than itself (CPU only).

Each building block is checked against a closed form, an invariant or a brute
force on tiny inputs, chosen so that a plausible slip (a dropped term, a wrong
sign, a transposed operand, a wrong head mapping, a swapped gate/up) fails.
The whole model is pinned by special cases whose result has a closed form.
"""

import math

import numpy as np
import pytest

from oracle import (OracleModel, argmax_lowest, attention_decode, rmsnorm, rope_apply,
                    rope_inv_freq, silu, softmax, top2_margin, weights_to_numpy)
from oracle.llama import rope_cos_sin
import synth
from synth import configs


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_form():
    x = np.array([3.0, 4.0])
    g = np.array([2.0, 0.5])
    r = math.sqrt((9 + 16) / 2)
    np.testing.assert_allclose(rmsnorm(x, g, 0.0), [2 * 3 / r, 0.5 * 4 / r], rtol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 64))
    y = rmsnorm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(rmsnorm(7.5 * x, np.ones(64), 0.0), y, rtol=1e-12)


def test_rmsnorm_eps_enters_inside_the_root():
    x = np.array([1e-3, -1e-3])
    eps = 1e-5
    np.testing.assert_allclose(rmsnorm(x, np.ones(2), eps), x / math.sqrt(1e-6 + eps), rtol=1e-14)


# ---------------------------------------------------------------- RoPE

def test_inv_freq_closed_form():
    np.testing.assert_allclose(rope_inv_freq(4, 10000.0), [1.0, 0.01], rtol=1e-15)
    f = rope_inv_freq(64, 500000.0)
    assert f[0] == 1.0
    np.testing.assert_allclose(f[-1], 500000.0 ** (-62 / 64), rtol=1e-14)


def test_llama3_scaling_regimes():
    base = rope_inv_freq(64, 500000.0)
    sc = rope_inv_freq(64, 500000.0, dict(factor=32.0, low_freq=1.0, high_freq=4.0, orig_max=8192))
    ratio = sc / base
    wavelen = 2 * math.pi / base
    short = wavelen < 8192 / 4
    long_ = wavelen > 8192 / 1
    assert short.any() and long_.any() and (~short & ~long_).any()
    np.testing.assert_allclose(ratio[short], 1.0, rtol=1e-15)
    np.testing.assert_allclose(ratio[long_], 1 / 32, rtol=1e-15)
    mid = ratio[~short & ~long_]
    assert np.all((mid > 1 / 32) & (mid < 1))
    # longer wavelengths are never scaled less than shorter ones
    assert np.all(np.diff(ratio) <= 1e-15)
    # the scaled frequencies still decrease with i
    assert np.all(np.diff(sc) < 0)


# Llama-3 frequency scaling at the Llama-3.2-1B setting (d = 64, theta = 5e5,
# factor 32, low-frequency factor 1, high-frequency factor 4, original context
# 8192), derived by hand from the published rule at 40-digit precision:
#   f_i = 5e5^(-2i/64);  wavelength wl_i = 2 pi / f_i;
#   wl < 8192/4 = 2048: keep f;  wl > 8192/1 = 8192: f/32;
#   else s = (8192/wl - 1) / (4 - 1) and f' = (1 - s) f/32 + s f.
#   i   f_i                      wl_i           8192/wl      s                 f'_i
#   14  3.21144599475259090e-3   1956.497       4.18707      (below 2048)      = f
#   15  2.13111953691196530e-3   2948.303       2.77854789   0.592849295003    1.29054792820926375e-3
#   16  1.41421356237309503e-3   4442.883       1.84384782   0.281282605163    4.29556796559368208e-4
#   17  9.38473870357380241e-4   6695.109       1.22357969   0.074526564161    9.70828780262767289e-5
#   18  6.22772421914595986e-4   10089.055      (above 8192)                   1.94616381848311246e-5
# (i = 16: f = 1/sqrt(5e5), so wl = 2 pi sqrt(5e5) = 4442.8829..., and
#  f' = f (0.718717/32 + 0.281283) = 0.303743 f.)
LLAMA3_BAND_GOLDEN = {
    14: 3.21144599475259090e-3,
    15: 1.29054792820926375e-3,
    16: 4.29556796559368208e-4,
    17: 9.70828780262767289e-5,
    18: 1.94616381848311246e-5,
}
# What three plausible misreadings of the band would give at i = 15, 16, 17:
# blending linearly in wavelength between the edges, blending the inverse
# frequency (harmonic) with the same weight, and swapping the two weights.
LLAMA3_BAND_MISREADINGS = {
    "blend in wavelength": {15: 1.82859762853031086e-3, 16: 8.80190766379930316e-4,
                            17: 2.50826798817474299e-4},
    "blend in 1/frequency": {15: 1.56450658892072502e-4, 16: 6.07473809782372115e-5,
                             17: 3.16094340067713531e-5},
    "weights swapped": {15: 9.07169094231200413e-4, 16: 1.02885093963788615e-3,
                        17: 8.70718300779771675e-4},
}
LLAMA3_SCALING = dict(factor=32.0, low_freq=1.0, high_freq=4.0, orig_max=8192)


def test_llama3_scaling_band_golden_values():
    sc = rope_inv_freq(64, 500000.0, LLAMA3_SCALING)
    for i, want in LLAMA3_BAND_GOLDEN.items():
        assert sc[i] == pytest.approx(want, rel=1e-13), i
    # every plausible misreading of the band misses the golden values by far
    for name, vals in LLAMA3_BAND_MISREADINGS.items():
        for i, wrong in vals.items():
            assert abs(wrong - LLAMA3_BAND_GOLDEN[i]) > 0.2 * LLAMA3_BAND_GOLDEN[i], (name, i)


def test_rope_half_split_pairs_and_sign():
    # d = 4: pair 0 is (x[0], x[2]); rotating e0 by +90 degrees gives e2
    x = np.array([1.0, 0.0, 0.0, 0.0])
    cos = np.array([0.0, 1.0])
    sin = np.array([1.0, 0.0])
    np.testing.assert_allclose(rope_apply(x, cos, sin), [0.0, 0.0, 1.0, 0.0], atol=1e-15)
    y = np.array([0.0, 0.0, 1.0, 0.0])
    np.testing.assert_allclose(rope_apply(y, cos, sin), [-1.0, 0.0, 0.0, 0.0], atol=1e-15)


def test_rope_identity_at_zero_and_norm_preserved():
    rng = np.random.default_rng(1)
    inv = rope_inv_freq(64, 500000.0)
    x = rng.normal(size=(3, 64))
    c0, s0 = rope_cos_sin([0], inv, np.float64)
    np.testing.assert_allclose(rope_apply(x, c0[0], s0[0]), x, rtol=0, atol=0)
    c, s = rope_cos_sin([1234], inv, np.float64)
    y = rope_apply(x, c[0], s[0])
    # every pair keeps its length
    np.testing.assert_allclose(y[:, :32] ** 2 + y[:, 32:] ** 2, x[:, :32] ** 2 + x[:, 32:] ** 2,
                               rtol=1e-12)


def test_rope_relative_position():
    rng = np.random.default_rng(2)
    inv = rope_inv_freq(64, 500000.0, dict(factor=32.0, low_freq=1.0, high_freq=4.0, orig_max=8192))
    q, k = rng.normal(size=64), rng.normal(size=64)

    def dot_at(m, n):
        cm, sm = rope_cos_sin([m], inv, np.float64)
        cn, sn = rope_cos_sin([n], inv, np.float64)
        return rope_apply(q, cm[0], sm[0]) @ rope_apply(k, cn[0], sn[0])

    assert dot_at(10, 3) == pytest.approx(dot_at(510, 503), rel=1e-9)
    assert dot_at(10, 3) != pytest.approx(dot_at(10, 4), rel=1e-3)


# ---------------------------------------------------------------- softmax, silu, argmax

def test_softmax_closed_form_and_invariants():
    np.testing.assert_allclose(softmax(np.array([0.0, math.log(3.0)])), [0.25, 0.75], rtol=1e-15)
    rng = np.random.default_rng(3)
    s = rng.normal(size=(4, 9)) * 5
    p = softmax(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(softmax(s + 100.0), p, rtol=1e-12)


def test_silu_values():
    assert silu(np.array(0.0)) == 0.0
    assert silu(np.array(1.0)) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    x = np.linspace(-6, 6, 13)
    np.testing.assert_allclose(silu(x) - silu(-x), x, rtol=1e-13, atol=1e-15)
    assert silu(np.array(40.0)) == pytest.approx(40.0, rel=1e-15)


def test_argmax_lowest_index_and_margin():
    v = np.array([[0.5, 2.0, -1.0, 2.0], [3.0, 3.0, 3.0, 1.0]])
    np.testing.assert_array_equal(argmax_lowest(v), [1, 0])
    np.testing.assert_allclose(top2_margin(np.array([[1.0, 4.0, 2.5]])), [1.5])


# ---------------------------------------------------------------- attention

def _attention_brute(q, K, V):
    """Explicit loops in Python floats, kv heads replicated up front."""
    Hq, d = q.shape
    T, Hkv, _ = K.shape
    rep = Hq // Hkv
    Kx = np.repeat(K, rep, axis=1)  # [T, Hq, d]; head h now sits at column h
    Vx = np.repeat(V, rep, axis=1)
    out = np.zeros((Hq, d))
    for h in range(Hq):
        scores = [sum(float(q[h, i]) * float(Kx[j, h, i]) for i in range(d)) / math.sqrt(d)
                  for j in range(T)]
        m = max(scores)
        e = [math.exp(s - m) for s in scores]
        z = sum(e)
        for i in range(d):
            out[h, i] = sum(e[j] / z * float(Vx[j, h, i]) for j in range(T))
    return out


def test_attention_brute_force():
    rng = np.random.default_rng(4)
    q = rng.normal(size=(4, 8))
    K = rng.normal(size=(5, 2, 8))
    V = rng.normal(size=(5, 2, 8))
    np.testing.assert_allclose(attention_decode(q, K, V), _attention_brute(q, K, V), rtol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(4, 8))
    V = rng.normal(size=(6, 2, 8))
    # one position: the output is that position's value
    np.testing.assert_allclose(attention_decode(q, rng.normal(size=(1, 2, 8)), V[:1]),
                               np.repeat(V[0], 2, axis=0), rtol=1e-14)
    # equal keys, or a zero query: the plain mean of the values
    K_eq = np.broadcast_to(rng.normal(size=(1, 2, 8)), (6, 2, 8))
    np.testing.assert_allclose(attention_decode(q, K_eq, V), np.repeat(V.mean(0), 2, axis=0),
                               rtol=1e-12)
    np.testing.assert_allclose(attention_decode(np.zeros((4, 8)), rng.normal(size=(6, 2, 8)), V),
                               np.repeat(V.mean(0), 2, axis=0), rtol=1e-12)


def test_attention_gqa_head_mapping():
    # query heads 0,1 read kv head 0 and heads 2,3 read kv head 1 (h // rep, not h % Hkv)
    V = np.zeros((3, 2, 4))
    V[:, 0, :] = 1.0
    V[:, 1, :] = 2.0
    o = attention_decode(np.ones((4, 4)), np.zeros((3, 2, 4)), V)
    np.testing.assert_allclose(o[:, 0], [1, 1, 2, 2])


def test_attention_scale_is_inverse_sqrt_d():
    d = 16
    q = np.zeros((1, d))
    q[0, 0] = 2.0
    K = np.zeros((2, 1, d))
    K[1, 0, 0] = 3.0
    V = np.zeros((2, 1, d))
    V[1, 0, 0] = 1.0
    s = 6.0 / math.sqrt(d)
    assert attention_decode(q, K, V)[0, 0] == pytest.approx(math.exp(s) / (1 + math.exp(s)),
                                                             rel=1e-14)


# ---------------------------------------------------------------- whole model

def _tiny_cfg(**kw):
    cfg = configs.model_config("tiny")
    cfg.update(kw)
    return cfg


def test_zero_layers_closed_form_logits_and_greedy_identity():
    """All layer matrices zero: x stays E[t], logits = E (E[t]/rms(E[t]) * g_f),
    and with random N(0, 0.02) embeddings the greedy id is the input token."""
    cfg = _tiny_cfg(norm_jitter=0.1)
    w = weights_to_numpy(synth.make_weights(cfg, zero_layers=True))
    m = OracleModel(cfg, w, np.float64)
    E = w["embed"].astype(np.float64)
    gf = w["final_norm"].astype(np.float64)
    toks = [5, 17, 4095, 0, 1234]
    seq = m.forward_sequence(toks)
    cache = m.new_cache()
    for p, t in enumerate(toks):
        e = E[t]
        want = E @ (e / np.sqrt(np.mean(e * e) + cfg["rms_eps"]) * gf)
        got = m.step(t, p, cache)
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(seq[p], want, rtol=1e-10, atol=1e-12)
        assert int(argmax_lowest(got)) == t


def test_untied_head_is_used():
    cfg = _tiny_cfg(tied=0)
    w = weights_to_numpy(synth.make_weights(cfg, zero_layers=True))
    m = OracleModel(cfg, w, np.float64)
    e = w["embed"][9].astype(np.float64)
    want = w["lm_head"].astype(np.float64) @ (e / np.sqrt(np.mean(e * e) + 1e-5))
    np.testing.assert_allclose(m.step(9, 0, m.new_cache()), want, rtol=1e-10)


def _one_layer(cfg, seed=0):
    cfg = dict(cfg, n_layers=1)
    return cfg, weights_to_numpy(synth.make_weights(cfg, seed=seed))


def test_uniform_attention_wiring():
    """W_q = 0 makes every softmax uniform over positions 0..p: the attention
    output of head h is the mean of v_{h // rep} over the prefix.  With the MLP
    zeroed the final residual has the closed form E[t_p] + W_o o_p."""
    cfg, w = _one_layer(_tiny_cfg(norm_jitter=0.1))
    w["wq"][0][:] = 0
    for k in ("w_gate", "w_up", "w_down"):
        w[k][0][:] = 0
    m = OracleModel(cfg, w, np.float64)
    toks = [3, 900, 77, 2048, 11, 5]
    Hq, Hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    E = w["embed"].astype(np.float64)
    n = np.stack([rmsnorm(E[t], w["attn_norm"][0].astype(np.float64), 1e-5) for t in toks])
    v = (n @ w["wv"][0].astype(np.float64).T).reshape(len(toks), Hkv, d)
    seq_logits = m.forward_sequence(toks)
    cache = m.new_cache()
    for p, t in enumerate(toks):
        vm = v[: p + 1].mean(0)  # [Hkv, d]
        o = np.concatenate([vm[h // (Hq // Hkv)] for h in range(Hq)])
        x = E[t] + w["wo"][0].astype(np.float64) @ o
        want = E @ rmsnorm(x, w["final_norm"].astype(np.float64), 1e-5)
        np.testing.assert_allclose(m.step(t, p, cache), want, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(seq_logits[p], want, rtol=1e-9, atol=1e-12)


def test_mlp_wiring_gate_and_up_not_swapped():
    """Attention output zeroed (W_o = 0); W_gate = c[I;0], W_up = [I;0],
    W_down = [I 0] gives x = E[t] + silu(c n) * n with n = RMSNorm(E[t]) g_mlp."""
    cfg, w = _one_layer(_tiny_cfg(norm_jitter=0.1))
    H, F = cfg["hidden"], cfg["ffn"]
    c = 3.0
    w["wo"][0][:] = 0
    eye = np.zeros((F, H), dtype=np.float32)
    eye[np.arange(H), np.arange(H)] = 1.0
    w["w_gate"][0] = c * eye
    w["w_up"][0] = eye.copy()
    w["w_down"][0] = eye.T.copy()
    m = OracleModel(cfg, w, np.float64)
    E = w["embed"].astype(np.float64)
    t = 321
    n = rmsnorm(E[t], w["mlp_norm"][0].astype(np.float64), 1e-5)
    x = E[t] + silu(c * n) * n
    want = E @ rmsnorm(x, w["final_norm"].astype(np.float64), 1e-5)
    np.testing.assert_allclose(m.step(t, 0, m.new_cache()), want, rtol=1e-9, atol=1e-12)


def test_token_by_token_equals_causal_sequence():
    cfg = _tiny_cfg(norm_jitter=0.1, rope_scaling=1, rope_factor=32.0, rope_low_freq=1.0,
                    rope_high_freq=4.0, rope_orig_max=8)
    w = weights_to_numpy(synth.make_weights(cfg))
    m = OracleModel(cfg, w, np.float64)
    toks = synth.prompt_tokens(cfg, 0, 11).numpy()
    seq = m.forward_sequence(toks, q_chunk=4)
    cache = m.new_cache()
    for p, t in enumerate(toks):
        np.testing.assert_allclose(m.step(int(t), p, cache), seq[p], rtol=1e-9, atol=1e-12)


def test_fp32_oracle_close_to_fp64():
    cfg = _tiny_cfg()
    w = weights_to_numpy(synth.make_weights(cfg))
    toks = synth.prompt_tokens(cfg, 0, 12).numpy()
    a = OracleModel(cfg, w, np.float32).forward_sequence(toks)
    b = OracleModel(cfg, w, np.float64).forward_sequence(toks)
    assert np.max(np.abs(a - b)) < 1e-4


def test_greedy_consistent_with_sequence():
    cfg = _tiny_cfg()
    w = weights_to_numpy(synth.make_weights(cfg))
    m = OracleModel(cfg, w, np.float64)
    prompt = synth.prompt_tokens(cfg, 0, 8).numpy()
    ids, lg = m.greedy(prompt, 6)
    full = np.concatenate([prompt, ids[:-1]])
    seq = m.forward_sequence(full, logits_at=np.arange(7, 7 + 7))
    np.testing.assert_allclose(np.stack(lg), seq, rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(argmax_lowest(seq), ids)
