"""The two matvec engines (mk_matvec_engine) against a float64 product of the
same bf16 weights, and their host-side argument checks."""

import ctypes

import pytest

import persistent_megakernel_02_b200 as mk
from persistent_megakernel_02_b200 import build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def test_engine_rejects_bad_requests_on_the_host():
    f = mk.lib().mk_matvec_engine
    p = ctypes.c_void_p(256)
    assert mk.STATUS[f(1, None, 128, 2048, p, 1, p, 0, 0, None)] == "MK_ERR_INVALID_ARG"
    assert mk.STATUS[f(1, p, 128, 2048, p, 9, p, 0, 0, None)] == "MK_ERR_UNSUPPORTED"     # nb > 8
    assert mk.STATUS[f(0, p, 128, 1024, p, 1, p, 0, 0, None)] == "MK_ERR_UNSUPPORTED"     # CUDA cores: K 2048
    assert mk.STATUS[f(1, p, 100, 2048, p, 1, p, 0, 0, None)] == "MK_ERR_UNSUPPORTED"     # rows % 128
    assert mk.STATUS[f(1, p, 128, 2000, p, 1, p, 0, 0, None)] == "MK_ERR_UNSUPPORTED"     # K % 64
    assert mk.STATUS[f(1, p, 128, 8192, p, 1, p, 0, 0, None)] == "MK_ERR_UNSUPPORTED"     # K > 4096
    assert mk.STATUS[f(2, p, 128, 2048, p, 1, p, 0, 0, None)] == "MK_ERR_INVALID_ARG"     # no such engine


@pytest.mark.gpu
@pytest.mark.parametrize("engine", ["cuda_cores", "tcgen05"])
@pytest.mark.parametrize("nb", [1, 3, 8])
@pytest.mark.parametrize("rows,K", [(1024, 2048), (4096, 2048), (768, 4096), (1024, 64)])
def test_engine_matches_float64(engine, nb, rows, K):
    import torch

    if engine == "cuda_cores" and K != 2048:
        pytest.skip("the CUDA-core engine streams 4-row pages of K = 2048")
    g = torch.Generator(device="cpu").manual_seed(1000 + rows + nb)
    W = (torch.randn(rows, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    X = torch.randn(nb, K, generator=g).float().cuda()
    Y = torch.full((nb, rows), float("nan"), device="cuda")
    mk.matvec_engine(engine, W, X, Y, wait_limit_ms=2000)
    mk.matvec_engine_status()
    ref = (X.double() @ W.double().t())
    err = (Y.double() - ref).abs().max().item()
    rel = ((Y.double() - ref).norm() / ref.norm()).item()
    assert torch.isfinite(Y).all()
    assert rel < 1e-5 and err < 1e-4 * ref.abs().max().item(), (engine, nb, rows, K, err, rel)
