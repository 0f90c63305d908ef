"""Host-side aggregation of the kernel's profile records (no GPU): the per-op
means, the per-(layer, op) windows, the layer chain and the per-SM spread that
persistent_megakernel_02_b200.profile.summarize derives from raw records."""

import numpy as np
import pytest

from persistent_megakernel_02_b200.profile import OPS, markdown, summarize

OP = {v: k for k, v in OPS.items()}


def _rec(op, layer, t_start, t_dep, t_done, t_sig, staged=0, last_warp=0, pages=0):
    r = np.zeros(32, dtype=np.int64)
    r[0] = OP[op] | (layer << 8) | (1 << 24)
    r[1], r[2], r[3], r[4] = t_start, t_dep, t_done, t_sig
    r[8] = pages
    r[11], r[12] = staged, last_warp
    return r


def _records():
    # two SMs, two layers of gate/up, then the LM head; times in ns
    rec = np.zeros((2, 3, 32), dtype=np.int64)
    rec[0, 0] = _rec("gu", 0, 1000, 1100, 5000, 5100, staged=1500, last_warp=5000, pages=4)
    rec[1, 0] = _rec("gu", 0, 1000, 1300, 7000, 7300, staged=1700, last_warp=7000, pages=4)
    rec[0, 1] = _rec("gu", 1, 8000, 8100, 9000, 9100, staged=8300, last_warp=9000, pages=4)
    rec[1, 1] = _rec("gu", 1, 8000, 8200, 9500, 9600, staged=8400, last_warp=9500, pages=4)
    rec[0, 2] = _rec("lm", 2, 10000, 10100, 20000, 20100, staged=10500, last_warp=20000, pages=8)
    rec[1, 2] = _rec("lm", 2, 10000, 10200, 22000, 22200, staged=10600, last_warp=22000, pages=8)
    return rec


def test_step_and_phase_windows():
    s = summarize(_records())
    assert s["step_us"] == pytest.approx((22200 - 1000) / 1e3)
    # gate/up windows: layer 0 from 1100 to 7300, layer 1 from 8100 to 9600
    assert s["phase_us_mean"]["gu"] == pytest.approx(((7300 - 1100) + (9600 - 8100)) / 2 / 1e3, abs=1e-3)
    assert s["phase_us_mean"]["lm"] == pytest.approx((22200 - 10100) / 1e3, abs=1e-3)


def test_per_op_means():
    d = summarize(_records())["per_op"]["gu"]
    assert d["n"] == 4
    waits = [1100 - 1000, 1300 - 1000, 8100 - 8000, 8200 - 8000]
    assert d["wait_us_mean"] == pytest.approx(np.mean(waits) / 1e3, abs=1e-3)
    stages = [1500 - 1100, 1700 - 1300, 8300 - 8100, 8400 - 8200]
    assert d["stage_us_mean"] == pytest.approx(np.mean(stages) / 1e3, abs=1e-3)
    assert d["pages_per_instr_mean"] == pytest.approx(4.0)


def test_chain_and_spread_use_the_middle_layers():
    s = summarize(_records())
    chain = s["chain_first_last_end_us"]
    # layers 0 and 1 are the middle pair of {0, 1, 2}; times from layer 0's first
    # QKV start, or from the first phase present when a layer has no QKV
    assert [c[:2] for c in chain] == [(0, "gu"), (1, "gu")]
    sp = s["spread_p0_10_50_90_100_us"]
    assert sp["lm"]["end"][0] == pytest.approx((20100 - 10100) / 1e3)
    assert sp["lm"]["end"][-1] == pytest.approx((22200 - 10100) / 1e3)
    assert sp["lm"]["end_by_sm"] == [10.0, 12.1]


def test_markdown_report_lists_every_op_present():
    text = markdown(summarize(_records()), bench_us=456.4)
    assert "bench without stamps: 456.4 us" in text
    rows = [ln for ln in text.splitlines() if ln.startswith("| gu ") or ln.startswith("| lm ")]
    assert len(rows) == 2
    assert "| 0 | gu |" in text and "| 1 | gu |" in text


def test_wait_share_of_the_sms_time():
    """Barrier waits (t_dep - t_start) and re-read time (summed over a CTA's 8
    warps) as shares of n_sm x step; page waits beside them."""
    rec = _records()
    rec[0, 0, 17] = 8 * 400    # 400 ns of re-reads per warp on SM 0's first instruction
    rec[1, 2, 7] = 8 * 1000    # 1000 ns of page waits per warp on SM 1's LM head
    s = summarize(rec)
    sm_time = 2 * (22200 - 1000)
    barrier = (100 + 300 + 100 + 200 + 100 + 200)
    assert s["wait_share"]["barrier"] == pytest.approx(barrier / sm_time, abs=1e-4)
    assert s["wait_share"]["data_poll"] == pytest.approx(400 / sm_time, abs=1e-4)
    assert s["wait_share"]["barrier_plus_poll"] == pytest.approx((barrier + 400) / sm_time, abs=1e-4)
    assert s["wait_share"]["page_wait"] == pytest.approx(1000 / sm_time, abs=1e-4)
    assert "Wait share" in markdown(s)
