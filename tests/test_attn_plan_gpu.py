"""The draft attention's split-KV planner (a device kernel run once per forward):
the chunk it picks from the actual context lengths, and the work list the
attention grid then runs."""
import random

import pytest
import torch

import synth
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def _plan(lens, valid, B, nkv, cap, chunk_min, slots):
    t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    v = torch.tensor(valid, dtype=torch.int32, device="cuda")
    return D.debug_attn_plan(t, v, B, nkv, cap, chunk_min, slots)


def _expected_items(lens, valid, B, nkv, chunk):
    items = []
    for r, (T, ok) in enumerate(zip(lens, valid)):
        q = -(-((T if ok else 0) + B) // chunk)
        items += [(r, g, c, T if ok else 0) for g in range(nkv) for c in range(q)]
    return items


@pytest.mark.parametrize("seed", range(6))
def test_plan_covers_every_chunk_once_in_grid_order(seed):
    rng = random.Random(seed)
    batch = rng.choice([1, 3, 32, 70, 200])
    B = rng.choice([4, 8, 16])
    nkv = rng.choice([2, 8])
    cap = rng.choice([512, 4096 + 2 * B, 32768 + 2 * B])
    lens = [rng.randint(0, cap - B) for _ in range(batch)]
    valid = [int(rng.random() > 0.1) for _ in range(batch)]
    chunk_min = 64 * rng.choice([1, 2, 4, 12, 28])
    chunk_min = max(chunk_min, 64 * -(-cap // (64 * 255)))  # at most 255 chunks a request
    slots = rng.choice([148, 296])
    chunk, items = _plan(lens, valid, B, nkv, cap, chunk_min, slots)
    assert chunk % 64 == 0 and chunk >= chunk_min
    assert items == _expected_items(lens, valid, B, nkv, chunk)


def test_plan_picks_the_measured_chunks():
    # 4 requests of 32768 keys, block 16, 148 resident CTAs (64 query rows per
    # kv head): nine chunks per request fill two waves (measured best)
    chunk, items = _plan([32768] * 4, [1] * 4, 16, 8, 32800, 1792, 148)
    assert -(-(32768 + 16) // chunk) == 9 and len(items) == 288
    # one request of 2048 keys, block 16: 256-512-key chunks (measured best)
    chunk, _ = _plan([2048], [1], 16, 8, 2080, 64, 148)
    assert 256 <= chunk <= 512, chunk
    # 32 requests uniform in [512, 4096], block 8, 296 resident CTAs (32 query
    # rows per kv head): 2240-2560-key chunks (the measured plateau)
    cfg = synth.get_config("qwen3_8b_bs32")
    lens = [int(x) for x in synth.make_ctx_lens(cfg)]
    chunk, _ = _plan(lens, [1] * len(lens), cfg.B, cfg.nkv, cfg.cache_cap, 1792, 296)
    assert 2240 <= chunk <= 2560, chunk


def test_plan_hook_rejects_bad_arguments():
    t = torch.zeros(4, dtype=torch.int32, device="cuda")
    L = D.lib()
    out = torch.zeros(4096, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    bad = [
        (4, 8, 8, 4096, 100, 296, 4096),    # chunk_min not a multiple of 64
        (4, 8, 8, 4096, 1024, 0, 4096),     # no slots
        (4, 8, 8, 4096, 1024, 296, 10),     # plan_out too short
        (0, 8, 8, 4096, 1024, 296, 4096),   # empty batch
    ]
    for batch, B, nkv, cap, cmin, slots, n in bad:
        assert L.dflash_debug_attn_plan(t.data_ptr(), t.data_ptr(), batch, B, nkv, cap, cmin, slots,
                                        out.data_ptr(), n, st) == D.EINVAL


def test_grid_slots_follow_occupancy():
    # two CTAs per SM for 32 query rows per kv head, one for 64 (measured)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert D.debug_attn_slots(128, 32, 8) == 2 * sms
    assert D.debug_attn_slots(128, 64, 16) == sms
