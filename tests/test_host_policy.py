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


def test_attention_plan_hook_validates_before_enqueueing(L):
    # every rejection happens on the host, before anything touches the (fake)
    # device pointers: a null pointer, sizes, a chunk that is not a positive
    # multiple of 64, more than 255 chunks or kv heads, a short or misaligned plan
    p = 4096  # never dereferenced on these paths
    bad = [
        (0, p, 4, 8, 8, 4096, 1024, 296, p, 4096),       # null ctx_len
        (p, p, 0, 8, 8, 4096, 1024, 296, p, 4096),       # empty batch
        (p, p, 4, 8, 256, 4096, 1024, 296, p, 4096),     # more than 255 kv heads
        (p, p, 4, 8, 8, 4096, 1000, 296, p, 4096),       # chunk_min not a multiple of 64
        (p, p, 4, 8, 8, 4096, 1024, 0, p, 4096),         # no resident slots
        (p, p, 4, 8, 8, 32768, 64, 296, p, 1 << 20),     # 512 chunks a request
        (p, p, 4, 8, 8, 4096, 1024, 296, p, 4 + 2 * 4 * 8 * 4 - 1),  # plan one int short
        (p, p, 4, 8, 8, 4096, 1024, 296, p + 4, 4096),   # plan not 8-byte aligned
        (p, p, 4, 8, 8, 4, 64, 296, p, 4096),            # cap below the block
    ]
    for ctx, valid, batch, B, nkv, cap, cmin, slots, out, n in bad:
        assert L.dflash_debug_attn_plan(ctx, valid, batch, B, nkv, cap, cmin, slots, out, n,
                                        None) == D.EINVAL
    assert L.dflash_debug_attn_slots(0, 32, 8) == D.EINVAL
    assert L.dflash_debug_attn_slots(128, 32, 0) == D.EINVAL
