"""The allocation-free greedy head against the decode step (needs a B200).

mk_greedy_head_noalloc serves callers that cannot allocate device memory on
their call path; its working memory is a static array inside the library.  Its
output must equal what mk_decode_step computes for the same hidden state.  With
every layer matrix zero, the decode step's final hidden state is exactly the
token's embedding row, so feeding that row to the head must reproduce the
step's logits and greedy ids -- checked on two calls in a row, each of which
reuses the scratch the previous one left behind.  Collected last, so a run that
stops at the first failure has run every other test first.
"""

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


def test_noalloc_head_rejects_oversized_requests():
    from persistent_megakernel_02_b200 import MkError, greedy_head_noalloc

    g = torch.ones(4096, dtype=torch.bfloat16, device="cuda")
    lm = torch.zeros((64, 4096), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(9, dtype=torch.int32, device="cuda")
    with pytest.raises(MkError, match="UNSUPPORTED"):  # 9 lanes: beyond the scratch array
        greedy_head_noalloc(torch.zeros((9, 64), device="cuda"), g[:64], lm[:, :64], 1e-5, ids)
    with pytest.raises(MkError, match="UNSUPPORTED"):  # 8 x 4096 floats: beyond the staging
        greedy_head_noalloc(torch.zeros((8, 4096), device="cuda"), g, lm, 1e-5, ids)
