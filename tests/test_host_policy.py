"""Host-side launch policies of the library, checked without a GPU (the
library loads and these calls touch no device memory)."""

import ctypes

import pytest

from block_diffusion_speculative_gemm_b200 import dflash as D


@pytest.fixture(scope="module")
def L():
    return D.lib()


@pytest.mark.parametrize("M,N,K", [(256, 6144, 4096), (256, 4096, 4096), (256, 24576, 4096),
                                   (256, 4096, 12288), (154, 4096, 20480), (154, 10240, 4096),
                                   (16, 24576, 4096), (1, 128, 64), (16384, 4096, 20480)])
def test_split_pick_is_a_count_the_gemm_runs_unchanged(L, M, N, K):
    s = L.dflash_debug_pick_splits(M, N, K)
    nkb = K // 64
    assert 1 <= s <= min(16, nkb)
    # every split but the last gets ceil(nkb / s) k-blocks and none is empty
    per = -(-nkb // s)
    assert -(-nkb // per) == s


def test_split_pick_rejects_bad_shapes(L):
    assert L.dflash_debug_pick_splits(0, 128, 64) == D.EINVAL
    assert L.dflash_debug_pick_splits(16, 128, 100) == D.EINVAL


def test_verify_workspace_covers_partials_and_grows_with_batch(L):
    V = 151936
    hdr = L.dflash_verify_workspace_size(0, 8, V)
    prev = hdr
    for b in (1, 2, 8, 32, 128, 1024):
        sz = L.dflash_verify_workspace_size(b, 8, V)
        assert sz % 256 == 0 and sz >= hdr + b * 8 * 8
        assert sz >= prev
        prev = sz


def test_test_hooks_reject_out_of_range_values(L):
    assert L.dflash_debug_attn_chunk(65) == D.EINVAL
    assert L.dflash_debug_attn_chunk(-64) == D.EINVAL
    assert L.dflash_debug_attn_chunk(0) == 0
    assert L.dflash_debug_gemm_mode(3) == D.EINVAL
    assert L.dflash_debug_gemm_mode(0) == 0
    assert L.dflash_debug_split_weight(ctypes.c_float(-1.0)) == D.EINVAL
    assert L.dflash_debug_split_weight(ctypes.c_float(4.0)) == 0
