"""Batched prefill on the tensor cores against the oracle and against the
token-by-token prefill (needs a B200).

mk_prefill runs every prompt token but the last through batched layers (tcgen05
GEMMs with the activations split into bf16 high and low parts, causal attention
over the paged cache) and the last one through the decode kernel.  Checked: the
last prompt position's logits and the teacher-forced decode steps that follow
(which read every K/V row the batched layers wrote) match the oracle within the
parity bounds; the batched and the token-by-token prefill agree closely; prompts
that span several 128-token tiles with a ragged tail, several 2048-token passes,
a prompt continued at start_pos > 0, and an fp16 KV cache.  The full-size
workloads (8192-token context, batch 4/8, 8B) take the batched path too, in
test_gpu_parity.py.
"""

import numpy as np
import pytest
import torch

import synth
from synth import configs
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from persistent_megakernel_02_b200 import build

    build.build()


def _mk(cfg, w, **kw):
    from persistent_megakernel_02_b200 import Megakernel

    return Megakernel(cfg, w, **kw)


def _prefill_then_steps(mk, cfg, prompt, teacher, chunks=None):
    """Prefill (in the given pieces), then teacher-forced steps: (last logits, step logits)."""
    V = cfg["vocab"]
    lg = torch.empty(V, dtype=torch.float32, device="cuda")
    pieces = chunks or [len(prompt)]
    p0 = 0
    for n in pieces:
        mk.prefill(0, [int(t) for t in prompt[p0:p0 + n]], start_pos=p0, logits_last=lg)
        p0 += n
    mk.sync()
    last = lg.cpu().numpy().copy()
    steps = []
    tok = torch.empty(1, dtype=torch.int32, device="cuda")
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    out = torch.empty((1, V), dtype=torch.float32, device="cuda")
    for t, tk in enumerate(teacher):
        tok.fill_(int(tk))
        mk.decode_step(tok, [len(prompt) + t], ids, out)
        mk.sync()
        steps.append(out[0].cpu().numpy().copy())
    return last, np.stack(steps)


def _against_oracle(cfg, w, prompt, teacher, last, steps, case):
    orc = H.oracle_for(cfg, w)
    w_last, w_steps = H.oracle_teacher_forced(orc, prompt, teacher, len(teacher))
    worst = H.compare_logits(last, w_last, f"{case} prefill")
    for t in range(len(teacher)):
        e = H.compare_logits(steps[t], w_steps[t], f"{case} step {t}")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    H.record(case, worst, len(teacher), 0)
    return worst


@pytest.mark.parametrize("wl,n_prompt", [("tiny", 300), ("tiny", 17), ("llama1b_bs1", 300)])
def test_batched_prefill_matches_oracle(wl, n_prompt):
    """17 tokens: the smallest batched prompt (16 batched + 1 decode step); 300:
    three 128-token tiles, the last ragged, and five 64-position KV pages."""
    cfg = configs.model_config(wl, max_batch=1, max_seq=n_prompt + 16)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, n_prompt).numpy()
    teacher = synth.teacher_tokens(cfg, 0, 8).numpy()
    mk = _mk(cfg, w)
    last, steps = _prefill_then_steps(mk, cfg, prompt, teacher)
    mk.close()
    _against_oracle(cfg, w, prompt, teacher, last, steps, f"batched prefill {wl} P={n_prompt}")


def test_batched_prefill_agrees_with_token_by_token():
    """The same prompt through both prefill paths: the KV rows differ only by
    summation order, so the last logits and the following steps agree far inside
    the parity bounds."""
    cfg = configs.model_config("llama1b_bs1", max_batch=1, max_seq=200)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 160).numpy()
    teacher = synth.teacher_tokens(cfg, 0, 6).numpy()
    got = []
    for tokenwise in (0, 1):
        mk = _mk(cfg, w, prefill_tokenwise=tokenwise)
        got.append(_prefill_then_steps(mk, cfg, prompt, teacher))
        mk.close()
    (lb, sb), (lt, stw) = got
    assert np.abs(lb - lt).max() < 2e-2
    assert np.abs(sb - stw).max() < 2e-2
    assert int(np.argmax(lb)) == int(np.argmax(lt)) or \
        abs(lt[int(np.argmax(lb))] - lt.max()) < 0.1


def test_batched_prefill_several_passes_and_a_ragged_last_one():
    """4100 tokens: 4099 run batched in passes of 2048, 2048 and 3 tokens (a pass
    of a single partial tile), then the last one through the decode kernel."""
    cfg = configs.model_config("tiny", max_batch=1, max_seq=4120)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 4100).numpy()
    teacher = synth.teacher_tokens(cfg, 0, 4).numpy()
    mk = _mk(cfg, w)
    last, steps = _prefill_then_steps(mk, cfg, prompt, teacher)
    mk.close()
    _against_oracle(cfg, w, prompt, teacher, last, steps, "batched prefill tiny P=4100 (3 passes)")


def test_prefill_continued_at_a_later_start_position():
    """A prompt prefilled in two calls (100 tokens, then 60 at start_pos 100):
    the second call's queries attend to the rows the first call wrote."""
    cfg = configs.model_config("tiny", max_batch=1, max_seq=200)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 160).numpy()
    teacher = synth.teacher_tokens(cfg, 0, 4).numpy()
    mk = _mk(cfg, w)
    last, steps = _prefill_then_steps(mk, cfg, prompt, teacher, chunks=[100, 60])
    mk.close()
    _against_oracle(cfg, w, prompt, teacher, last, steps, "batched prefill tiny 100+60")


def test_batched_prefill_fp16_cache_and_untied_random_gains():
    cfg = configs.model_config("tiny", max_batch=1, max_seq=220, kv_dtype=1, tied=0, norm_jitter=0.2)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 200).numpy()
    teacher = synth.teacher_tokens(cfg, 0, 4).numpy()
    mk = _mk(cfg, w)
    last, steps = _prefill_then_steps(mk, cfg, prompt, teacher)
    mk.close()
    _against_oracle(cfg, w, prompt, teacher, last, steps, "batched prefill tiny fp16 KV, untied")


def test_prefill_into_a_second_slot_leaves_the_first_intact():
    """Slot 1's batched prefill writes only slot 1's pages: slot 0's decode steps
    after it still match the oracle."""
    cfg = configs.model_config("tiny", max_batch=2, max_seq=160)
    w = H.gpu_weights(cfg)
    p0 = synth.prompt_tokens(cfg, 0, 90).numpy()
    p1 = synth.prompt_tokens(cfg, 1, 130).numpy()
    teacher = [synth.teacher_tokens(cfg, b, 4).numpy() for b in range(2)]
    mk = _mk(cfg, w)
    pre, lg, _ = H.run_teacher_forced(mk, cfg, [p0, p1], teacher, 4)
    mk.close()
    orc = H.oracle_for(cfg, w)
    for b, pr in enumerate([p0, p1]):
        w_pre, w_steps = H.oracle_teacher_forced(orc, pr, teacher[b], 4)
        H.compare_logits(pre[b], w_pre, f"slot {b} prefill")
        for t in range(4):
            H.compare_logits(lg[t, b], w_steps[t], f"slot {b} step {t}")
