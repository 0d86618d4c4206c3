"""Vocabulary-parallel LM head and verify: the oracle's shard records, merged in
shard order, give the whole row's argmax (lowest id on ties) and softmax
max-probability (pinned against scipy's softmax and NumPy's first argmax), for
uneven shards and for ties planted on shard boundaries.  The two-rank gloo
test runs the exchange of the multi-GPU driver on the host: every rank gathers
every rank's records in rank order and merges to the same result."""

import os
import socket

import numpy as np
import pytest
import scipy.special
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from block_diffusion_speculative_gemm_b200 import vocab_parallel as VP

VPO = O.vocab_parallel


@pytest.mark.parametrize("V,world", [(10, 1), (10, 3), (151936, 8), (7, 7), (1000, 6)])
def test_shard_bounds_cover_the_vocabulary_in_order(V, world):
    b = VP.shard_bounds(V, world)
    assert b[0][0] == 0 and b[-1][1] == V and len(b) == world
    assert all(b[k][1] == b[k + 1][0] for k in range(world - 1))
    sizes = [hi - lo for lo, hi in b]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def _rows(V, seed):
    rng = np.random.default_rng(seed)
    L = rng.normal(0, 3, size=(6, V))
    L[1, :] = 0.0                     # every entry tied: id 0, probability 1 / V
    L[2, [V // 3, 2 * V // 3]] = 50.0  # an exact tie across a shard boundary: the lower id
    L[3, V - 1] = 60.0                 # the maximum in the last shard
    return L


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_merged_records_equal_the_whole_row(world):
    V = 997
    L = _rows(V, world)
    b = VP.shard_bounds(V, world)
    p = scipy.special.softmax(L, axis=1)
    for r in range(L.shape[0]):
        tok, conf = VPO.merge_records([VPO.shard_record(L[r], lo, hi) for lo, hi in b])
        assert tok == int(np.argmax(L[r]))
        np.testing.assert_allclose(conf, p[r].max(), rtol=1e-12)
        assert VPO.merge_argmax([VPO.verify_shard_record(L[r], lo, hi) for lo, hi in b]) == tok
    assert VPO.merge_records([VPO.shard_record(L[2], lo, hi) for lo, hi in b])[0] == V // 3


def _port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        V = 1003
        L = _rows(V, 11)
        lo, hi = VP.shard_bounds(V, world)[rank]
        # this rank's records as the library lays them out: (max, id bits, sum, 0)
        rec = torch.zeros((L.shape[0], 4), dtype=torch.float32)
        for r in range(L.shape[0]):
            m, i, s = VPO.shard_record(L[r], lo, hi)
            rec[r, 0], rec[r, 2] = m, s
            rec[r, 1] = torch.tensor([i], dtype=torch.int32).view(torch.float32)[0]
        g = VP.all_gather()(rec)
        assert tuple(g.shape) == (world, L.shape[0], 4)
        got = []
        for r in range(L.shape[0]):
            recs = [(float(g[k, r, 0]), int(g[k, r, 1:2].view(torch.int32)[0]), float(g[k, r, 2]))
                    for k in range(world)]
            got.append(VPO.merge_records(recs))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_records_in_rank_order():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank, args=(2, _port(), out), nprocs=2, join=True, start_method="spawn")
    L = _rows(1003, 11)
    want = [VPO.merge_records([VPO.shard_record(L[r], 0, 1003)]) for r in range(L.shape[0])]
    for rank in (0, 1):
        toks = [t for t, _ in out[rank]]
        assert toks == [t for t, _ in want]
        np.testing.assert_allclose([c for _, c in out[rank]], [c for _, c in want], rtol=1e-5)
