"""The shared seeded input generator: determinism, range, distribution (CPU)."""

import numpy as np
import torch

import synth
from synth import configs


def _mix32_py(x):
    x &= 0xFFFFFFFF
    x ^= x >> 16
    x = (x * 0x7FEB352D) & 0xFFFFFFFF
    x ^= x >> 15
    x = (x * 0x846CA68B) & 0xFFFFFFFF
    x ^= x >> 16
    return x


def test_mix32_matches_plain_integer_arithmetic():
    xs = [0, 1, 2, 0xFFFFFFFF, 0x12345678, 0x80000000, 987654321]
    got = synth.mix32(torch.tensor(xs, dtype=torch.int64)).tolist()
    assert got == [_mix32_py(x) for x in xs]


def test_normal_is_deterministic_and_distinct_per_tensor():
    a = synth.normal_bf16((1000, 64), seed=0, tensor_id=5)
    b = synth.normal_bf16((1000, 64), seed=0, tensor_id=5)
    c = synth.normal_bf16((1000, 64), seed=0, tensor_id=6)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a, c)
    # a prefix of a larger draw is the smaller draw (element counter, not shape)
    d = synth.normal_bf16((64000,), seed=0, tensor_id=5)
    assert torch.equal(d[:64000].view(1000, 64), a)


def test_normal_statistics():
    x = synth.normal_bf16((1 << 20,), seed=3, tensor_id=11).float().numpy()
    assert abs(x.mean()) < 1e-4
    assert abs(x.std() / 0.02 - 1) < 0.01
    # Irwin-Hall n=4 excess kurtosis is -0.3
    k = np.mean((x - x.mean()) ** 4) / x.var() ** 2 - 3
    assert -0.4 < k < -0.2


def test_tokens_range_and_spread():
    t = synth.tokens(100000, 128256, seed=1)
    assert t.dtype == torch.int32
    assert int(t.min()) >= 0 and int(t.max()) < 128256
    assert len(torch.unique(t)) > 50000


def test_step_bytes_llama1b():
    cfg = configs.model_config("llama1b_bs1")
    wb = configs.weight_bytes(cfg)
    assert abs(wb / 1e9 - 2.4716) < 0.001
    assert configs.kv_bytes_per_pos(cfg) == 32 * 1024
