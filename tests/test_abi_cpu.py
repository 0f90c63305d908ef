"""The C-ABI library on the host (no GPU): exports, tape lowering and simulation,
fault detection by the simulator, and host-side argument checks."""

import ctypes
import os
import re

import pytest

import persistent_megakernel_02_b200 as mk
from persistent_megakernel_02_b200 import build
from synth import configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "mk.h")).read()
    return sorted(set(re.findall(r"^\s*(?:mk_status|const char\*)\s+(mk_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert {"mk_create", "mk_decode_step", "mk_prefill", "mk_destroy"} <= set(names)
    lib = ctypes.CDLL(build.LIB)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(mk._SIGS), "binding misses a declared entry point"


def test_version_string():
    assert "megakernel" in mk.version()


@pytest.mark.parametrize("wl", list(configs.WORKLOADS))
@pytest.mark.parametrize("n_sm", [148, 132, 37])
@pytest.mark.parametrize("dyn", [0, 25])
def test_tapes_are_deadlock_free_and_cover_every_output(wl, n_sm, dyn):
    cfg = configs.model_config(wl)
    for nb in sorted({1, cfg["max_batch"]}):
        r = mk.plan_check(cfg, n_sm, nb, dyn_percent=dyn)
        assert r["deadlock_free"] and r["coverage_ok"] and r["targets_ok"], (wl, n_sm, nb, r)
        # bytes per SM balanced to within one attention slice + one page
        assert r["bytes_max_sm"] - r["bytes_min_sm"] <= 2 * 16384 * (1 + 130 // r["attn_slices"])
        assert r["ring_pages"] >= 8


def test_ring_depth_follows_the_measured_rule():
    """The deepest ring that fits (228 KiB carveout) only for HBM-streamed shapes with
    a small activation region (the 1B shape at batch 1); the 196 KiB carveout for
    the rest (batch 4 and 8, the 8B shape, an L2-resident model)."""
    want = {"llama1b_bs1": 13, "llama1b_long": 13, "llama1b_bs4": 9, "llama1b_bs8": 9,
            "llama8b_bs1": 10, "tiny": 11}
    for wl, pages in want.items():
        r = mk.plan_check(configs.model_config(wl), 148, 1)
        assert r["ring_pages"] == pages, (wl, r["ring_pages"])
        assert r["smem_bytes"] <= 232448


def test_ragged_shapes_lower_cleanly():
    cfg = configs.model_config("tiny", vocab=4099, ffn=1000, max_batch=3, max_seq=77)
    for nb in (1, 2, 3):
        r = mk.plan_check(cfg, 148, nb)
        assert r["deadlock_free"] and r["coverage_ok"] and r["targets_ok"]


@pytest.mark.parametrize("fault", [1, 2])
def test_simulator_reports_planted_faults(fault):
    """1: a dropped signal, 2: a wait target one too high -- both leave SMs stuck."""
    r = mk.plan_check(configs.model_config("tiny"), 148, 1, fault=fault)
    assert not r["deadlock_free"]
    assert not r["targets_ok"]


def test_simulator_reports_an_uncovered_claim_range():
    """3: one SM's copy of the LM head's claim range ends a row block early; the
    ranges of the pool then disagree and the simulator reports the coverage."""
    r = mk.plan_check(configs.model_config("tiny"), 148, 1, fault=3, dyn_percent=25)
    assert r["deadlock_free"] and r["targets_ok"]
    assert not r["coverage_ok"]


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(hidden=4104), dict(n_heads=12, n_kv_heads=4),
                                 dict(max_batch=9), dict(ffn=1001), dict(n_kv_heads=3),
                                 dict(kv_dtype=2), dict(max_batch=8, hidden=4096)])
def test_unsupported_configs_are_rejected(bad):
    cfg = configs.model_config("tiny", **bad)
    with pytest.raises(mk.MkError, match="UNSUPPORTED"):
        mk.plan_check(cfg, 148, 1)


def test_create_rejects_missing_weights_before_touching_the_gpu():
    c = mk.config_struct(configs.model_config("tiny"))
    w = mk.MkWeights()  # all NULL
    h = ctypes.c_void_p()
    st = mk.lib().mk_create(ctypes.byref(c), ctypes.byref(w), None, ctypes.byref(h))
    assert mk.STATUS[st] == "MK_ERR_INVALID_ARG"


def _fake_weights(cfg):
    """Non-null, 16-byte aligned placeholders: enough for mk_create's host checks,
    never dereferenced before the device checks."""
    L = cfg["n_layers"]
    arrs = [(ctypes.c_void_p * L)(*([4096] * L)) for _ in range(9)]
    w = mk.MkWeights(embed=4096, lm_head=None if cfg["tied"] else 4096, final_norm=4096,
                     **{n: ctypes.cast(a, mk._PP) for n, a in zip(mk.Megakernel._LAYER, arrs)})
    return w, arrs


@pytest.mark.parametrize("field,value", [("tensor_core_units", 5), ("tensor_core_units", -1), ("region_cut", 2),
                                         ("dyn_percent", 91), ("ring_pages", -1)])
def test_create_rejects_out_of_range_options_before_touching_the_gpu(field, value):
    cfg = configs.model_config("tiny")
    c = mk.config_struct(cfg)
    w, _keep = _fake_weights(cfg)
    h = ctypes.c_void_p()
    o = mk.MkOptions(**{field: value})
    assert mk.STATUS[mk.lib().mk_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(o), ctypes.byref(h))] \
        == "MK_ERR_INVALID_ARG"


def test_create_accepts_the_options_range_up_to_the_device_checks():
    import torch

    if torch.cuda.is_available():
        pytest.skip("placeholder weight pointers: the accepted case would reach the device")
    cfg = configs.model_config("tiny")
    c = mk.config_struct(cfg)
    w, _keep = _fake_weights(cfg)
    for kw in ({}, {"tensor_core_units": 4}, {"region_cut": 1}, {"dyn_percent": 90}):
        h = ctypes.c_void_p()
        o = mk.MkOptions(**kw)
        st = mk.STATUS[mk.lib().mk_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(o), ctypes.byref(h))]
        assert st == "MK_ERR_CUDA", (kw, st)  # past every host check: no device here


def test_noalloc_head_rejects_bad_arguments_on_the_host():
    f = mk.lib().mk_greedy_head_noalloc
    ids = ctypes.c_void_p(16)
    assert mk.STATUS[f(None, 1, 64, ids, ids, 10, 1e-5, None, ids, None)] == "MK_ERR_INVALID_ARG"
    assert mk.STATUS[f(ids, 0, 64, ids, ids, 10, 1e-5, None, ids, None)] == "MK_ERR_INVALID_ARG"
    assert mk.STATUS[f(ids, 9, 64, ids, ids, 10, 1e-5, None, ids, None)] == "MK_ERR_UNSUPPORTED"
    assert mk.STATUS[f(ids, 8, 4096, ids, ids, 10, 1e-5, None, ids, None)] == "MK_ERR_UNSUPPORTED"


def test_library_rope_frequencies_match_the_published_rule():
    """The inverse frequencies the library builds its RoPE table from equal the
    hand-derived Llama-3 band values (oracle pins) and the oracle's own, on the
    1B shape (scaled) and the 8B shape (unscaled, d = 128)."""
    from oracle import rope_inv_freq as oracle_inv_freq
    from tests.test_oracle_pins import LLAMA3_BAND_GOLDEN, LLAMA3_SCALING

    lib_f = mk.rope_inv_freq(configs.model_config("llama1b_bs1"))
    for i, want in LLAMA3_BAND_GOLDEN.items():
        assert lib_f[i] == pytest.approx(want, rel=1e-13), i
    for wl, scaling in (("llama1b_bs1", LLAMA3_SCALING), ("llama8b_bs1", None), ("tiny", None)):
        cfg = configs.model_config(wl)
        got = mk.rope_inv_freq(cfg)
        want = oracle_inv_freq(cfg["head_dim"], cfg["rope_theta"], scaling)
        assert got == pytest.approx(list(want), rel=1e-13), wl


def test_rope_inv_freq_rejects_bad_arguments():
    cfg = configs.model_config("llama1b_bs1")
    c = mk.config_struct(cfg)
    out = (ctypes.c_double * 32)()
    assert mk.lib().mk_rope_inv_freq(ctypes.byref(c), out, 31) == 1
    bad = dict(cfg, rope_high_freq=0.5)
    assert mk.lib().mk_rope_inv_freq(ctypes.byref(mk.config_struct(bad)), out, 32) == 1


def test_noalloc_head_binding_rejects_bad_tensors_before_launch():
    """The C entry point sees raw pointers only; the binding refuses a wrong dtype,
    a wrong shape, a non-contiguous operand, a short ids buffer and host tensors
    before anything reaches the library (CPU tensors: nothing can launch)."""
    import torch

    from persistent_megakernel_02_b200 import MkError, greedy_head_noalloc

    H, V, nb = 64, 128, 2
    hidden = torch.zeros((nb, H), dtype=torch.float32)
    gain = torch.ones(H, dtype=torch.bfloat16)
    lm = torch.zeros((V, H), dtype=torch.bfloat16)
    ids = torch.zeros(nb, dtype=torch.int32)
    cases = {
        "hidden dtype": (hidden.to(torch.bfloat16), gain, lm, ids, None),
        "gain dtype": (hidden, gain.float(), lm, ids, None),
        "lm_head non-contiguous": (hidden, gain, torch.zeros((H, V), dtype=torch.bfloat16).t(), ids, None),
        "lm_head wrong width": (hidden, gain, torch.zeros((V, H + 8), dtype=torch.bfloat16), ids, None),
        "lm_head sliced": (hidden, gain, torch.zeros((V, 2 * H), dtype=torch.bfloat16)[:, :H], ids, None),
        "ids short": (hidden, gain, lm, ids[:1], None),
        "ids dtype": (hidden, gain, lm, ids.long(), None),
        "logits shape": (hidden, gain, lm, ids, torch.zeros((nb, V + 1))),
        "host tensors": (hidden, gain, lm, ids, torch.zeros((nb, V))),
    }
    for what, (h, g, w, i, lg) in cases.items():
        with pytest.raises(MkError, match="INVALID_ARG"):
            greedy_head_noalloc(h, g, w, 1e-5, i, lg)


@pytest.mark.parametrize("wl", list(configs.WORKLOADS))
def test_region_cut_tapes_are_deadlock_free_and_split_the_outputs(wl):
    """The two launches of the region cut: the layers tape produces every layer
    output once and no LM-head tile, the LM-head tape every LM-head tile once and
    nothing else, each deadlock-free with exact wait targets."""
    cfg = configs.model_config(wl)
    for nb in sorted({1, cfg["max_batch"]}):
        for region in (1, 2):
            r = mk.plan_check(cfg, 148, nb, region=region)
            assert r["deadlock_free"] and r["coverage_ok"] and r["targets_ok"], (wl, nb, region, r)
    whole = mk.plan_check(cfg, 148, 1)
    layers = mk.plan_check(cfg, 148, 1, region=1)
    lm = mk.plan_check(cfg, 148, 1, region=2)
    assert layers["n_instr_total"] + lm["n_instr_total"] == whole["n_instr_total"]


def test_plan_check_rejects_an_unknown_region():
    c = mk.config_struct(configs.model_config("tiny"))
    rep = mk.MkPlanReport()
    assert mk.lib().mk_plan_check(ctypes.byref(c), 148, 1, 0, 0, 3, 0, ctypes.byref(rep)) == 1
    assert mk.lib().mk_plan_check(ctypes.byref(c), 148, 1, 0, 0, 0, 5, ctypes.byref(rep)) == 1


def test_default_tensor_core_units_are_gate_up_and_lm_head():
    """The measured default (tensor_core_units 0) runs gate/up and the LM head as
    tensor-core units with 5-8 lanes, and nothing with 1-4 lanes: its tapes equal the
    explicit selections."""
    cfg = configs.model_config("llama1b_bs8")
    keys = ("n_instr_total", "bytes_min_sm", "bytes_max_sm")
    pick = lambda nb, u: tuple(mk.plan_check(cfg, 148, nb, tensor_core_units=u)[k] for k in keys)
    assert pick(8, 0) == pick(8, 4) != pick(8, 1)
    assert pick(5, 0) == pick(5, 4)
    assert pick(4, 0) == pick(4, 1)


def test_gate_up_blocks_stay_out_of_the_cumulative_balance():
    """The 128 gate/up tensor-core blocks (32 pages each, fewer than the SMs) must not
    tilt the other phases: the SMs that hold one carry its 32 pages on top of an even
    share of everything else, so the step's per-SM bytes spread by at least a block."""
    cfg = configs.model_config("llama1b_bs8")
    page = 16384
    cuda_cores = mk.plan_check(cfg, 148, 8, tensor_core_units=1)
    gu = mk.plan_check(cfg, 148, 8, tensor_core_units=3)
    assert cuda_cores["bytes_max_sm"] - cuda_cores["bytes_min_sm"] <= 2 * page
    assert gu["bytes_max_sm"] - gu["bytes_min_sm"] >= 32 * page


@pytest.mark.parametrize("units", [2, 3, 4])
@pytest.mark.parametrize("region", [0, 1, 2])
def test_tensor_core_unit_tapes_cover_their_blocks(units, region):
    """With 5-8 lanes the Llama-3.2-1B-shaped kernel can run the LM head (2), gate/up
    (3) or both (4) as 128-row tensor-core blocks: every block once, the CUDA-core
    form of the same op not at all, deadlock-free, in each region of a cut too; 1-4
    lanes keep the CUDA-core ops."""
    cfg = configs.model_config("llama1b_bs8")
    for nb in (8, 5, 4, 1):
        r = mk.plan_check(cfg, 148, nb, region=region, tensor_core_units=units)
        assert r["deadlock_free"] and r["coverage_ok"] and r["targets_ok"], (units, region, nb, r)
