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


@pytest.mark.parametrize("N,K,M", [
    (128, 64, 16),          # one tile, one k-block: fewer iterations than workers
    (6144, 4096, 256),      # QKV projection: ~20 k-blocks per worker, tiles split 3-4 ways
    (4096, 4096, 256),      # output projection
    (24576, 4096, 256),     # SwiGLU gate/up
    (4096, 12288, 256),     # down projection
    (1000, 512, 133),       # ragged weight and token rows
    (4096, 20480, 154),     # injection fc over five taps
    (640, 320, 1100),       # several token tiles, the last ragged
    (130, 128, 48),         # the last weight tile has 2 live rows
    (151936 // 8, 512, 224),  # an LM-head-like width
])
@pytest.mark.parametrize("mode", ["single", "pair"])
def test_stream_k_gemm_matches_float64(N, K, M, mode):
    """Stream-K: every worker streams the same number of k-blocks; split tiles
    are finished inside the kernel by their last piece, summing the pieces in
    worker order.  The product must be the fp64 product, and two runs must be
    bit-identical (the sum order does not depend on which piece arrives last)."""
    D.debug_gemm_mode(MODES[mode][1])
    W, X = _inputs(N, K, M, N + 3 * K + M, torch.float16)
    Wd, Xd = W.cuda(), X.cuda()
    out, err = D.debug_gemm_streamk(Wd, Xd)
    again, err2 = D.debug_gemm_streamk(Wd, Xd)
    assert err == 0 and err2 == 0
    ref = X.double() @ W.double().T
    scale = ref.abs().max().item()
    assert (out.double().cpu() - ref).abs().max().item() <= 2e-5 * scale + 1e-6
    assert torch.equal(out, again)
