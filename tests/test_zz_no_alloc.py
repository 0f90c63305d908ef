"""The allocation-free greedy head against the decode step (needs a B200).

mk_greedy_head_noalloc serves callers that cannot allocate device memory on
their call path; its working memory is a static array inside the library.  Its
output must equal what mk_decode_step computes for the same hidden state.  With
every layer matrix zero, the decode step's final hidden state is exactly the
token's embedding row, so feeding that row to the head must reproduce the
step's logits and greedy ids -- checked on two calls in a row, each of which
reuses the scratch the previous one left behind.  Random hidden states are
checked against a float64 norm + matvec + argmax (8 lanes of 2048, which needs
the >48 KiB shared-memory staging), and an exact tie between rows that different
blocks stream must go to the lower row.  Collected last, so a run that stops at
the first failure has run every other test first.
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


@pytest.mark.parametrize("wl,nb", [("tiny", 2), ("llama1b_bs1", 1)])
def test_noalloc_head_matches_decode_step(wl, nb):
    from persistent_megakernel_02_b200 import Megakernel, greedy_head_noalloc

    cfg = configs.model_config(wl, max_batch=nb, max_seq=16)
    w = synth.make_weights(cfg, device="cuda", zero_layers=True)
    mk = Megakernel(cfg, w)
    V = cfg["vocab"]
    for call, base in enumerate((11, 2900)):  # two calls in a row
        toks = [(base + 977 * b) % V for b in range(nb)]
        tok = torch.tensor(toks, dtype=torch.int32, device="cuda")
        ids_ref = torch.empty(nb, dtype=torch.int32, device="cuda")
        lg_ref = torch.empty((nb, V), dtype=torch.float32, device="cuda")
        mk.decode_step(tok, [call] * nb, ids_ref, lg_ref)
        mk.sync()
        hidden = w["embed"][tok.long()].float().contiguous()
        ids = torch.full((nb,), -1, dtype=torch.int32, device="cuda")
        lg = torch.empty((nb, V), dtype=torch.float32, device="cuda")
        greedy_head_noalloc(hidden, w["final_norm"], w["embed"], cfg["rms_eps"], ids, lg)
        torch.cuda.synchronize()
        for b in range(nb):
            H.compare_logits(lg[b].cpu().numpy(), lg_ref[b].cpu().numpy(), f"call {call} lane {b}")
        assert ids.tolist() == ids_ref.tolist() == toks
    mk.close()


def _f64_head(hidden, gain, lm, eps):
    """float64 RMSNorm (gain applied) + LM-head matvec of every lane."""
    x = hidden.double().cpu().numpy()
    g = gain.double().cpu().numpy()
    W = lm.double().cpu().numpy()
    n = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g
    return n @ W.T


def test_noalloc_head_random_hidden_matches_float64():
    from persistent_megakernel_02_b200 import greedy_head_noalloc

    nb, H, V = 8, 2048, 32000
    lm = synth.normal_bf16((V, H), 3, 11, device="cuda")
    gain = (synth.normal_bf16((H,), 3, 12, std=0.2, device="cuda").float() + 1.0).to(torch.bfloat16)
    hidden = synth.normal_bf16((nb, H), 3, 13, std=1.5, device="cuda").float().contiguous()
    for call in range(2):  # two calls in a row share the scratch array
        ids = torch.full((nb,), -1, dtype=torch.int32, device="cuda")
        lg = torch.empty((nb, V), dtype=torch.float32, device="cuda")
        greedy_head_noalloc(hidden, gain, lm, 1e-5, ids, lg)
        torch.cuda.synchronize()
        want = _f64_head(hidden, gain, lm, 1e-5)
        got = lg.cpu().numpy()
        assert np.abs(got - want).max() < 1e-4, f"call {call}"
        for b in range(nb):
            top = np.sort(want[b])[-2:]
            if top[1] - top[0] > 1e-3:
                assert ids[b].item() == int(np.argmax(want[b])), (call, b)
        hidden = -hidden  # the second call sees a different state


def test_noalloc_head_ties_across_blocks_take_the_lowest_row():
    """Rows 100 and 25000 (and 7 and 30000) are identical, and the hidden state
    is that row, so the two logits tie exactly at the top; the rows are streamed
    by different blocks, and the lower row must win whichever one is the copy."""
    from persistent_megakernel_02_b200 import greedy_head_noalloc

    H, V = 2048, 32000
    lm = synth.normal_bf16((V, H), 5, 21, device="cuda")
    lm[25000] = lm[100]
    lm[7] = lm[30000]
    gain = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    hidden = torch.stack([lm[100], lm[30000]]).float().contiguous()
    ids = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    lg = torch.empty((2, V), dtype=torch.float32, device="cuda")
    greedy_head_noalloc(hidden, gain, lm, 1e-5, ids, lg)
    torch.cuda.synchronize()
    assert lg[0, 100].item() == lg[0, 25000].item()
    assert lg[1, 7].item() == lg[1, 30000].item()
    assert ids.tolist() == [100, 7]


def test_noalloc_head_rejects_oversized_requests():
    from persistent_megakernel_02_b200 import MkError, greedy_head_noalloc

    g = torch.ones(4096, dtype=torch.bfloat16, device="cuda")
    lm = torch.zeros((64, 4096), dtype=torch.bfloat16, device="cuda")
    g64 = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    lm64 = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(9, dtype=torch.int32, device="cuda")
    with pytest.raises(MkError, match="UNSUPPORTED"):  # 9 lanes: beyond the scratch array
        greedy_head_noalloc(torch.zeros((9, 64), device="cuda"), g64, lm64, 1e-5, ids)
    with pytest.raises(MkError, match="UNSUPPORTED"):  # 8 x 4096 floats: beyond the staging
        greedy_head_noalloc(torch.zeros((8, 4096), device="cuda"), g, lm, 1e-5, ids)
