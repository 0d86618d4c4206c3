"""tcgen05 GEMM core against a float64 matrix product (torch CPU matmul)."""

import pytest
import torch

from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu

# weight layout and launch shape: row-major weights through a tensor map (single
# CTAs), or the pre-tiled image with single CTAs or CTA pairs (cta_group::2)
MODES = {"rowmajor": (False, 0), "single": (True, 1), "pair": (True, 2)}


@pytest.fixture(autouse=True)
def _reset_mode():
    yield
    D.debug_gemm_mode(0)


def _inputs(N, K, M, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * 0.05).to(dtype)
    X = torch.randn(M, K, generator=g).to(dtype)
    return W, X


@pytest.mark.parametrize("N,K,M,splits", [
    (128, 64, 16, 1),        # one tile, one k-block
    (384, 256, 32, 1),
    (256, 4096, 256, 4),     # full token tile, split-K
    (1000, 512, 133, 3),     # ragged weight rows and token rows
    (512, 1024, 300, 2),     # two token tiles, ragged second one
    (128, 192, 1, 5),        # one token row, more splits than fit evenly
    (6144, 4096, 256, 3),    # QKV projection of the 8B-shaped draft
    (640, 320, 64, 2),       # five weight tiles: the last pair has one live half
    (130, 128, 48, 1),       # two weight tiles, the second with 2 live rows
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", list(MODES))
def test_gemm_matches_float64(N, K, M, splits, dtype, mode):
    tiled, launch = MODES[mode]
    D.debug_gemm_mode(launch)
    W, X = _inputs(N, K, M, N * 7 + K + M, dtype)
    err = D.new_workspace(256)
    out = D.debug_gemm(W.cuda(), X.cuda(), splits, err, tiled=tiled)
    torch.cuda.synchronize()
    assert D.get_error(err) == 0
    got = out.double().sum(0).cpu()
    ref = X.double() @ W.double().T
    scale = ref.abs().max().item()
    assert (got - ref).abs().max().item() <= 2e-5 * scale + 1e-6
    # every split holds the product over its own K range
    if out.shape[0] > 1:
        per = -(-(K // 64) // out.shape[0])
        k1 = min(K, per * 64)
        ref0 = X[:, :k1].double() @ W[:, :k1].double().T
        assert (out[0].double().cpu() - ref0).abs().max().item() <= 2e-5 * scale + 1e-6


@pytest.mark.parametrize("N,K,M", [(1024, 256, 40), (151936 // 16, 512, 224), (2000, 128, 96)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", list(MODES))
def test_lmhead_epilogue_stats(N, K, M, dtype, mode):
    tiled, launch = MODES[mode]
    D.debug_gemm_mode(launch)
    W, X = _inputs(N, K, M, N + K + M, dtype)
    err = D.new_workspace(256)
    stats, logits = D.debug_lmhead(W.cuda(), X.cuda(), err, tiled=tiled)
    torch.cuda.synchronize()
    assert D.get_error(err) == 0
    ref = (X.double() @ W.double().T)
    scale = ref.abs().max().item()
    lg = logits.double().cpu()
    assert (lg - ref).abs().max().item() <= 2e-5 * scale
    st = stats.double().cpu()
    idx = stats.view(torch.int32)[:, :, 1].long().cpu()
    tiles = st.shape[1]
    for t in range(tiles):
        blk = lg[:, t * 128:(t + 1) * 128]
        mx, ix = blk.max(dim=1)
        # stats are computed from the kernel's own fp32 logits: exact max and first argmax
        assert torch.equal(st[:, t, 0], mx)
        first = (blk == mx[:, None]).double().argmax(dim=1) + t * 128
        assert torch.equal(idx[:, t], first.long())
        se = torch.exp(blk - mx[:, None]).sum(1)
        assert torch.allclose(st[:, t, 2], se, rtol=1e-5)
