"""GPU path vs the CPU oracle, through the C ABI (needs a B200).

Every test builds seeded bf16 weights on the GPU, runs the persistent kernel via
mk_prefill / mk_decode_step, and compares logits (max-abs <= 5e-2, rel-L2 <=
1e-2 per step and sequence) and greedy ids (identical where the oracle's top-2
margin exceeds 0.1) with the oracle on the same inputs.
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


def _teacher_forced_case(wl, n_steps=None, nb=None, mk_kw=None, **cfg_over):
    wlc = configs.WORKLOADS[wl]
    cfg = configs.model_config(wl, **cfg_over)
    nb = nb or wlc["batch"]
    n_steps = n_steps or wlc["decode_steps"]
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, wlc["prompt_lens"][b]).numpy() for b in range(nb)]
    teacher = [synth.teacher_tokens(cfg, b, n_steps).numpy() for b in range(nb)]
    mk = _mk(cfg, w, **(mk_kw or {}))
    pre, lg, ids = H.run_teacher_forced(mk, cfg, prompts, teacher, n_steps)
    mk.close()
    orc = H.oracle_for(cfg, w)
    worst = (0.0, 0.0)
    checked = 0
    for b in range(nb):
        w_pre, w_steps = H.oracle_teacher_forced(orc, prompts[b], teacher[b], n_steps)
        e = H.compare_logits(pre[b], w_pre, f"{wl} lane {b} prefill")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        for t in range(n_steps):
            e = H.compare_logits(lg[t, b], w_steps[t], f"{wl} lane {b} step {t}")
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
            checked += H.compare_ids(ids[t, b], w_steps[t], f"{wl} lane {b} step {t}")
    tag = ",".join(f"{k}={v}" for k, v in sorted({**cfg_over, **(mk_kw or {})}.items()))
    H.record(f"{wl}[{tag}] x{nb} lanes" if tag else f"{wl} x{nb} lanes", worst, n_steps, checked)
    return worst, checked


def test_tiny_teacher_forced():
    worst, checked = _teacher_forced_case("tiny")
    assert checked > 0
    print("tiny worst", worst)


def test_tiny_random_norm_gains_and_untied():
    _teacher_forced_case("tiny", norm_jitter=0.2, tied=0)


def test_tiny_fp16_kv_cache():
    _teacher_forced_case("tiny", kv_dtype=1)


def test_tiny_ragged_vocab_and_ffn():
    # vocab 4099 leaves a short last LM-head unit; ffn 1000 needs 5 down-proj K slices
    _teacher_forced_case("tiny", vocab=4099, ffn=1000)


@pytest.mark.parametrize("kvh", [2, 1])
def test_tiny_head_dim_128_short_context(kvh):
    # 128-dim heads over a one-page context: each SM takes one query head of a KV
    # group (two threads per output dim pair of a run of positions in P.V)
    _teacher_forced_case("tiny", head_dim=128, n_kv_heads=kvh)


def test_tiny_batch_of_three_lanes():
    cfg = configs.model_config("tiny", max_batch=3, max_seq=64)
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, n).numpy() for b, n in enumerate([5, 9, 17])]
    teacher = [synth.teacher_tokens(cfg, b, 12).numpy() for b in range(3)]
    mk = _mk(cfg, w)
    pre, lg, ids = H.run_teacher_forced(mk, cfg, prompts, teacher, 12)
    mk.close()
    orc = H.oracle_for(cfg, w)
    for b in range(3):
        w_pre, w_steps = H.oracle_teacher_forced(orc, prompts[b], teacher[b], 12)
        H.compare_logits(pre[b], w_pre)
        for t in range(12):
            H.compare_logits(lg[t, b], w_steps[t], f"lane {b} step {t}")
            H.compare_ids(ids[t, b], w_steps[t])


@pytest.mark.parametrize("lens", [[300], [520, 130]])
def test_tiny_long_context_split_attention(lens):
    """Contexts of several KV pages are split over SMs and merged (online-softmax
    partials); lanes of one step use different splits."""
    nb = len(lens)
    cfg = configs.model_config("tiny", max_batch=nb, max_seq=max(lens) + 8)
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, n).numpy() for b, n in enumerate(lens)]
    teacher = [synth.teacher_tokens(cfg, b, 6).numpy() for b in range(nb)]
    mk = _mk(cfg, w)
    pre, lg, ids = H.run_teacher_forced(mk, cfg, prompts, teacher, 6)
    mk.close()
    orc = H.oracle_for(cfg, w)
    for b in range(nb):
        w_pre, w_steps = H.oracle_teacher_forced(orc, prompts[b], teacher[b], 6)
        H.compare_logits(pre[b], w_pre, f"lane {b} prefill")
        for t in range(6):
            H.compare_logits(lg[t, b], w_steps[t], f"lane {b} step {t}")
            H.compare_ids(ids[t, b], w_steps[t])


@pytest.mark.parametrize("lens", [[600], [700, 300]])
def test_tiny_head_dim_128_merges_many_slices(lens):
    """128-dim heads over contexts of 19-22 KV pages: a (lane, kv head) runs as 9 or more
    slices, and the last one merges them through shared-memory weights; a lane with 10
    pages (5 slices) merges by the per-thread walk in the same step."""
    nb = len(lens)
    cfg = configs.model_config("tiny", max_batch=nb, max_seq=max(lens) + 8, head_dim=128)
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, n).numpy() for b, n in enumerate(lens)]
    teacher = [synth.teacher_tokens(cfg, b, 6).numpy() for b in range(nb)]
    mk = _mk(cfg, w)
    pre, lg, ids = H.run_teacher_forced(mk, cfg, prompts, teacher, 6)
    mk.close()
    orc = H.oracle_for(cfg, w)
    worst = (0.0, 0.0)
    checked = 0
    for b in range(nb):
        w_pre, w_steps = H.oracle_teacher_forced(orc, prompts[b], teacher[b], 6)
        e = H.compare_logits(pre[b], w_pre, f"lane {b} prefill")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        for t in range(6):
            e = H.compare_logits(lg[t, b], w_steps[t], f"lane {b} step {t}")
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
            checked += H.compare_ids(ids[t, b], w_steps[t])
    H.record(f"tiny[head_dim=128] contexts {lens} x{nb} lanes", worst, 6, checked)


def test_tiny_free_run_greedy_chained_on_device():
    wlc = configs.WORKLOADS["tiny"]
    cfg = configs.model_config("tiny")
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 8).numpy()
    n = wlc["decode_steps"]
    mk = _mk(cfg, w)
    first = mk.prefill(0, [int(t) for t in prompt])
    ids = torch.tensor([first], dtype=torch.int32, device="cuda")
    got = [first]
    for t in range(n):
        mk.decode_step(ids, [8 + t], ids)  # the step reads its token from the ids buffer
        got.append(int(ids.item()))
    mk.sync()
    mk.close()
    orc = H.oracle_for(cfg, w)
    want, want_logits = orc.greedy(prompt, n)
    for t in range(n + 1):
        from oracle import top2_margin

        if float(top2_margin(want_logits[t])) <= H.MARGIN:
            break  # beyond a near-tie the two runs may legitimately diverge
        assert got[t] == want[t], f"step {t}: {got[t]} != {want[t]}"


def test_multi_step_launch_matches_single_steps_and_oracle():
    """mk_decode_steps runs n chained greedy steps in one launch; its logits equal
    n launches of mk_decode_step, and its ids follow the oracle's greedy run."""
    cfg = configs.model_config("tiny", max_batch=3, max_seq=48)
    w = H.gpu_weights(cfg)
    lens = [5, 8, 11]
    prompts = [synth.prompt_tokens(cfg, b, n).tolist() for b, n in enumerate(lens)]
    n, V = 10, cfg["vocab"]
    # multi-step: prefill every slot, one launch of n steps (lanes at different positions)
    mk = _mk(cfg, w)
    first = [mk.prefill(b, prompts[b]) for b in range(3)]
    tok = torch.tensor(first, dtype=torch.int32, device="cuda")
    ids = torch.empty((n, 3), dtype=torch.int32, device="cuda")
    lg = torch.empty((n, 3, V), dtype=torch.float32, device="cuda")
    mk.decode_steps(tok, lens, n, ids, lg)
    mk.sync()
    mk.close()
    # the same steps one launch at a time
    mk1 = _mk(cfg, w)
    for b in range(3):
        assert mk1.prefill(b, prompts[b]) == first[b]
    cur = torch.tensor(first, dtype=torch.int32, device="cuda")
    out1 = torch.empty(3, dtype=torch.int32, device="cuda")
    lg1 = torch.empty((3, V), dtype=torch.float32, device="cuda")
    for t in range(n):
        mk1.decode_step(cur, [p + t for p in lens], out1, lg1)
        mk1.sync()
        np.testing.assert_allclose(lg[t].cpu().numpy(), lg1.cpu().numpy(), atol=2e-3, rtol=0)
        assert out1.tolist() == ids[t].tolist()
        cur.copy_(out1)
    mk1.close()
    # and the oracle's own greedy run, up to its first near-tie
    from oracle import top2_margin

    orc = H.oracle_for(cfg, w)
    for b in range(3):
        want, want_lg = orc.greedy(np.array(prompts[b]), n)
        got = [first[b]] + ids[:, b].tolist()
        for t in range(n + 1):
            if float(top2_margin(want_lg[t])) <= H.MARGIN:
                break
            assert got[t] == want[t], (b, t)


@pytest.mark.parametrize("dyn", [25, 90])
def test_tiny_dynamic_tails_teacher_forced(dyn):
    """Gate/up, down and LM-head rows partly claimed at run time (ragged shapes: a
    short last LM-head unit, 5 down K slices) still match the oracle."""
    worst, checked = _teacher_forced_case("tiny", mk_kw=dict(dyn_percent=dyn), vocab=4099, ffn=1000)
    assert checked > 0


def test_dynamic_tails_give_the_static_logits_bit_for_bit():
    """Which SM computes a row does not change its value: every output row is one
    warp's sum and the residual accumulators are fixed point, so the logits and ids
    of a chained multi-step launch are identical with and without claims."""
    cfg = configs.model_config("tiny", max_batch=3, max_seq=48)
    w = H.gpu_weights(cfg)
    lens = [5, 8, 11]
    prompts = [synth.prompt_tokens(cfg, b, n).tolist() for b, n in enumerate(lens)]
    n, V = 8, cfg["vocab"]
    runs = []
    for dyn in (0, 40):
        mk = _mk(cfg, w, dyn_percent=dyn)
        first = [mk.prefill(b, prompts[b]) for b in range(3)]
        tok = torch.tensor(first, dtype=torch.int32, device="cuda")
        ids = torch.empty((n, 3), dtype=torch.int32, device="cuda")
        lg = torch.empty((n, 3, V), dtype=torch.float32, device="cuda")
        mk.decode_steps(tok, lens, n, ids, lg)
        mk.sync()
        mk.close()
        runs.append((first, ids.cpu().numpy(), lg.cpu().numpy()))
    assert runs[0][0] == runs[1][0]
    np.testing.assert_array_equal(runs[0][1], runs[1][1])
    np.testing.assert_array_equal(runs[0][2], runs[1][2])


def test_greedy_ties_take_the_lowest_row_across_sms():
    """Exact ties in the LM head: with every row identical all logits are equal and
    the greedy id is row 0; with the first half of the rows negated, the winner is
    row 0 or the first row of the second half (whichever half has the larger
    logit), rows that other SMs stream."""
    cfg = configs.model_config("tiny", tied=0, max_seq=32)
    w = H.gpu_weights(cfg)
    V = cfg["vocab"]
    row = w["lm_head"][17].clone()
    w["lm_head"][:] = row
    prompt = synth.prompt_tokens(cfg, 0, 6).tolist()
    lg = torch.empty(V, dtype=torch.float32, device="cuda")
    mk = _mk(cfg, w)
    first = mk.prefill(0, prompt, logits_last=lg)
    mk.sync()
    mk.close()
    vals = lg.cpu().numpy()
    assert np.all(vals == vals[0]), "identical rows must give identical logits"
    assert first == 0
    m = V // 2 + 3
    w["lm_head"][:m] = -row
    mk = _mk(cfg, w)
    first = mk.prefill(0, prompt, logits_last=lg)
    mk.sync()
    mk.close()
    vals = lg.cpu().numpy()
    want = m if vals[m] > vals[0] else 0
    assert vals[0] != vals[m]
    assert first == want, (first, want, vals[0], vals[m])


def test_multi_step_launch_across_the_attention_mode_threshold():
    """Contexts of at most 4 KV pages use single-head attention units, longer ones
    split the pages over slices and merge; one multi-step launch over positions
    250..261 changes mode at 256 from one step to the next.  Its logits match the
    oracle at every step."""
    cfg = configs.model_config("tiny", max_batch=1, max_seq=280)
    w = H.gpu_weights(cfg)
    prompt = synth.prompt_tokens(cfg, 0, 250).tolist()
    teacher = synth.teacher_tokens(cfg, 0, 12).numpy()
    n, V = 12, cfg["vocab"]
    mk = _mk(cfg, w)
    mk.prefill(0, prompt)  # itself crosses 64-position pages, not the threshold
    tok = torch.tensor([int(teacher[0])], dtype=torch.int32, device="cuda")
    ids = torch.empty((n, 1), dtype=torch.int32, device="cuda")
    lg = torch.empty((n, 1, V), dtype=torch.float32, device="cuda")
    mk.decode_steps(tok, [250], n, ids, lg)  # positions 250..261: 4 pages of 64 end at 255
    mk.sync()
    mk.close()
    orc = H.oracle_for(cfg, w)
    greedy = [int(teacher[0])] + ids[:, 0].tolist()
    _, w_steps = H.oracle_teacher_forced(orc, np.array(prompt), np.array(greedy[:n]), n)
    for t in range(n):
        H.compare_logits(lg[t, 0].cpu().numpy(), w_steps[t], f"step {t} (position {250 + t})")


def test_zero_layers_greedy_is_identity_tiny():
    cfg = configs.model_config("tiny")
    w = H.gpu_weights(cfg, zero_layers=True)
    mk = _mk(cfg, w)
    toks = [3, 4095, 17, 0, 2222]
    ids, lg = mk.decode_step_host([toks[0]], [0], want_logits=True)
    assert ids[0] == toks[0]
    for p, t in enumerate(toks[1:], start=1):
        ids, _ = mk.decode_step_host([t], [p])
        assert ids[0] == t
    mk.close()


def test_llama1b_bs1_teacher_forced_full():
    worst, checked = _teacher_forced_case("llama1b_bs1")
    print("llama1b_bs1 worst", worst, "ids checked", checked)
    assert checked > 20


@pytest.mark.slow
@pytest.mark.parametrize("wl", ["llama1b_long", "llama1b_bs4", "llama1b_bs8", "llama8b_bs1"])
def test_full_size_workloads_teacher_forced(wl):
    """The long-context (8192-token KV, 64 steps), batch-4/8 (prompts 512..1408,
    128 steps) and 8B (2048-token prompt, 128 steps) workloads at full size and
    full length: every lane's prompt is prefilled, then every decode step the
    workload names is compared with the oracle's causal pass."""
    worst, checked = _teacher_forced_case(wl)
    print(wl, "worst", worst, "ids checked", checked)
    assert checked > 0


def test_llama1b_zero_layers_identity_full_size():
    cfg = configs.model_config("llama1b_bs1")
    w = H.gpu_weights(cfg, zero_layers=True)
    mk = _mk(cfg, w)
    toks = synth.prompt_tokens(cfg, 0, 6).tolist()
    for p, t in enumerate(toks):
        ids, _ = mk.decode_step_host([t], [p])
        assert ids[0] == t
    mk.close()


def test_batch_lane_matches_single_sequence():
    """Lane i of a batch-4 step equals sequence i run alone (same slot contents)."""
    cfg = configs.model_config("tiny", max_batch=4, max_seq=48)
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, 6 + 3 * b).numpy() for b in range(4)]
    teacher = [synth.teacher_tokens(cfg, b, 6).numpy() for b in range(4)]
    mk = _mk(cfg, w)
    _, lg4, _ = H.run_teacher_forced(mk, cfg, prompts, teacher, 6)
    mk.close()
    for b in range(4):
        mk1 = _mk(cfg, w)
        _, lg1, _ = H.run_teacher_forced(mk1, cfg, [prompts[b]], [teacher[b]], 6)
        mk1.close()
        np.testing.assert_allclose(lg4[:, b], lg1[:, 0], atol=2e-3, rtol=0)


def test_bounded_wait_times_out_and_context_survives():
    """A wait whose target can never be met ends with MK_ERR_TIMEOUT after the
    configured limit; the context stays usable and a fresh handle works."""
    cfg = configs.model_config("tiny")
    w = H.gpu_weights(cfg)
    bad = _mk(cfg, w, wait_limit_ms=100, debug_fault=1)
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad.decode_step(tok, [0], ids)
    st = bad.status()
    from persistent_megakernel_02_b200 import STATUS

    assert STATUS[st] == "MK_ERR_TIMEOUT", bad.error_string()
    # later steps return at once while the error is pending
    bad.decode_step(tok, [1], ids)
    assert STATUS[bad.status()] in ("MK_ERR_TIMEOUT", "MK_ERR_ABORTED")
    bad.close()
    torch.cuda.synchronize()
    good = _mk(cfg, w)
    ids_h, _ = good.decode_step_host([5], [0])
    good.close()
    assert 0 <= ids_h[0] < cfg["vocab"]


def test_invalid_arguments_are_rejected_on_the_host():
    from persistent_megakernel_02_b200 import MkError

    cfg = configs.model_config("tiny")
    w = H.gpu_weights(cfg)
    mk = _mk(cfg, w)
    with pytest.raises(MkError, match="INVALID_ARG"):
        mk.prefill(0, [1, 2, cfg["vocab"]])
    with pytest.raises(MkError, match="INVALID_ARG"):
        mk.decode_step_host([1], [cfg["max_seq"]])
    with pytest.raises(MkError, match="INVALID_ARG"):
        mk.prefill(1, [1])  # slot beyond max_batch
    mk.close()


def test_out_of_range_device_token_is_reported():
    from persistent_megakernel_02_b200 import STATUS

    cfg = configs.model_config("tiny")
    w = H.gpu_weights(cfg)
    mk = _mk(cfg, w)
    tok = torch.tensor([cfg["vocab"] + 7], dtype=torch.int32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    mk.decode_step(tok, [0], ids)
    assert STATUS[mk.status()] == "MK_ERR_DEVICE_FAULT"
    mk.clear_error()
    tok.fill_(3)
    mk.decode_step(tok, [0], ids)
    assert STATUS[mk.status()] == "MK_OK"
    mk.close()


@pytest.mark.parametrize("wl,nb", [("tiny", 3), ("llama1b_bs1", 1)])
def test_region_cut_gives_the_single_launch_results_bit_for_bit(wl, nb):
    """Two launches per step (layers, then the LM head) compute exactly what one
    launch does: the same code per output row and fixed-point residuals, so a
    chained multi-step run and a token-by-token prefill give identical logits and
    ids with and without the cut."""
    cfg = configs.model_config(wl, max_batch=nb, max_seq=64)
    w = H.gpu_weights(cfg)
    lens = [5 + 3 * b for b in range(nb)]
    prompts = [synth.prompt_tokens(cfg, b, n).tolist() for b, n in enumerate(lens)]
    n, V = 6, cfg["vocab"]
    runs = []
    for cut in (0, 1):
        mk = _mk(cfg, w, region_cut=cut, prefill_tokenwise=1)
        lg0 = torch.empty(V, dtype=torch.float32, device="cuda")
        first = [mk.prefill(b, prompts[b], logits_last=lg0) for b in range(nb)]
        tok = torch.tensor(first, dtype=torch.int32, device="cuda")
        ids = torch.empty((n, nb), dtype=torch.int32, device="cuda")
        lg = torch.empty((n, nb, V), dtype=torch.float32, device="cuda")
        mk.decode_steps(tok, lens, n, ids, lg)
        mk.sync()
        mk.close()
        runs.append((first, lg0.cpu().numpy(), ids.cpu().numpy(), lg.cpu().numpy()))
    assert runs[0][0] == runs[1][0]
    np.testing.assert_array_equal(runs[0][1], runs[1][1])
    np.testing.assert_array_equal(runs[0][2], runs[1][2])
    np.testing.assert_array_equal(runs[0][3], runs[1][3])


@pytest.mark.parametrize("nb,units", [(8, 4), (5, 4), (8, 2)])
def test_tensor_core_units_match_oracle_and_cuda_cores(nb, units):
    """5-8 lanes run the 8-lane kernel, whose gate/up and LM head can run on tcgen05
    tensor cores (128-row blocks, accumulators in tensor memory).  A 2-layer model
    of the Llama-3.2-1B shape with a ragged vocabulary (32001 rows: the last block
    holds one row) matches the oracle at every teacher-forced step, and the same
    handle on CUDA cores only within summation-order differences."""
    cfg = configs.model_config("llama1b_bs8", max_batch=8, max_seq=96, n_layers=2, vocab=32001)
    w = H.gpu_weights(cfg)
    prompts = [synth.prompt_tokens(cfg, b, 20 + 7 * b).numpy() for b in range(nb)]
    teacher = [synth.teacher_tokens(cfg, b, 6).numpy() for b in range(nb)]
    runs = []
    for sel in (units, 1):  # the tensor-core units asked for, then none
        mk = _mk(cfg, w, tensor_core_units=sel)
        runs.append(H.run_teacher_forced(mk, cfg, prompts, teacher, 6))
        mk.close()
    (pre, lg, ids), (pre_cc, lg_cc, _) = runs
    np.testing.assert_allclose(lg, lg_cc, atol=5e-3, rtol=0)
    orc = H.oracle_for(cfg, w)
    worst, checked = (0.0, 0.0), 0
    for b in range(nb):
        w_pre, w_steps = H.oracle_teacher_forced(orc, prompts[b], teacher[b], 6)
        H.compare_logits(pre[b], w_pre, f"lane {b} prefill")
        for t in range(6):
            e = H.compare_logits(lg[t, b], w_steps[t], f"lane {b} step {t}")
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
            checked += H.compare_ids(ids[t, b], w_steps[t], f"lane {b} step {t}")
    H.record(f"tensor-core units {units}, 2-layer 1B shape, vocab 32001, x{nb} lanes", worst, 6, checked)
