"""Vocabulary-parallel drafting and verify on one GPU, the ranks emulated as
separate shard models and workspaces whose calls run one after another (no
kernel waits for another): per step every rank's forward, then the records
stacked in rank order (what the all-gather delivers), then every rank's
commit.

* Verify: the merged accept equals dflash_verify on the whole logits, bit for
  bit, including ties planted on shard boundaries.
* Drafting: every rank ends with the same block, equal to the whole-vocabulary
  draft, and the oracle's draft rules hold.
"""

import numpy as np
import pytest
import torch

import synth
from synth.configs import shrink
from tests.gpu_common import DraftReport, built, check_draft_request, max_pos_for, oracle_caches_from
from block_diffusion_speculative_gemm_b200 import dflash as D
from block_diffusion_speculative_gemm_b200 import vocab_parallel as VP

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("b,B,world,dtype", [(32, 8, 8, "bf16"), (5, 4, 3, "f32"),
                                             (128, 16, 2, "bf16")])
def test_verify_over_vocabulary_shards_matches_verify(b, B, world, dtype):
    V = 151936
    case = synth.make_verify_case(b, B, V, f"vp_{b}_{B}", plant=("uniform",), dtype=dtype,
                                  adversarial=True)
    logits = case["logits"].cuda()
    bounds = VP.shard_bounds(V, world)
    # exact ties across every shard boundary in request 0's rows
    for lo, hi in bounds[1:]:
        logits[0, :, lo] = logits[0, :, lo - 1] = 1e3
    draft = case["draft"].cuda()
    cap = 3 * B

    def outs():
        return dict(out=torch.full((b, cap), -1, dtype=torch.int32, device="cuda"),
                    ol=torch.zeros(b, dtype=torch.int32, device="cuda"),
                    seq=torch.full((b,), 50, dtype=torch.int32, device="cuda"),
                    acc=torch.zeros(b, dtype=torch.int32, device="cuda"),
                    nxt=torch.zeros(b, dtype=torch.int32, device="cuda"))

    ref, got = outs(), outs()
    ws = D.new_workspace(D.verify_workspace_size(b, B, V))
    D.verify(logits, draft, ref["out"], ref["ol"], ref["seq"], ref["acc"], ref["nxt"], ws)
    recs = []
    for lo, hi in bounds:
        shard = logits[:, :, lo:hi].contiguous()
        mine = torch.empty((b * B, 2), dtype=torch.float32, device="cuda")
        D.verify_shard(shard, lo, mine, ws)
        recs.append(mine)
    D.verify_merge(torch.stack(recs), draft, V, got["out"], got["ol"], got["seq"], got["acc"],
                   got["nxt"], ws)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def _emulated_draft(models, wss, anchors, ctx, kc, vc, B, steps, batch):
    """Runs the step calls of every emulated rank, exchanging records by stacking."""
    for m, ws in zip(models, wss):
        D.draft_begin(m, anchors, ctx, kc.shape[3], B, steps, ws)
    for t in range(steps):
        rows = D.draft_rows(batch, B, steps, t)
        recs = []
        for m, ws in zip(models, wss):
            mine = torch.empty((rows, 4), dtype=torch.float32, device="cuda")
            D.draft_forward_shard(m, ctx, kc, vc, B, steps, t, mine, ws)
            recs.append(mine)
        gathered = torch.stack(recs)
        for m, ws in zip(models, wss):
            D.draft_commit_shards(m, gathered, batch, B, steps, t, ws)
    res = []
    for m, ws in zip(models, wss):
        out = torch.full((batch, B), -5, dtype=torch.int32, device="cuda")
        cst = torch.full((batch, B), -5, dtype=torch.int32, device="cuda")
        D.draft_end(m, B, steps, out, ws, commit_step=cst)
        res.append((out, cst))
    torch.cuda.synchronize()
    for ws in wss:
        assert D.get_error(ws) == 0
    return [(o.cpu(), c.cpu()) for o, c in res]


@pytest.mark.parametrize("name,world", [("small", 3), ("qwen3_8b_bs32", 2)])
def test_draft_over_vocabulary_shards_matches_the_whole_draft(name, world):
    if name == "small":
        base = synth.get_config("qwen3_8b_bs32")
        cfg = shrink(base, L=2, V=4099, batch=5, ctx=("uniform", 30, 700), I=1024, d=1024,
                     H_t=512).replace(name="vp8b")
    else:
        cfg = synth.get_config(name)
    b = built(cfg)
    ctx = synth.make_ctx_lens(cfg).cuda()
    anchors = synth.make_anchors(cfg).cuda()
    kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
    kc, vc = kc.cuda(), vc.cuda()
    # the whole-vocabulary draft
    whole = torch.zeros((cfg.batch, cfg.B), dtype=torch.int32, device="cuda")
    wcst = torch.zeros((cfg.batch, cfg.B), dtype=torch.int32, device="cuda")
    ws0 = b.model.workspace(cfg.batch, cfg.B, 0)
    D.draft_block(b.model, anchors, ctx, kc, vc, cfg.B, cfg.steps, whole, ws0, commit_step=wcst)
    # world = 1 through the driver: the step calls give the one-call draft
    one = torch.zeros_like(whole)
    VP.draft_block(b.model, anchors, ctx, kc, vc, cfg.B, cfg.steps, one, ws0,
                   gather=lambda x: x[None])
    torch.cuda.synchronize()
    assert torch.equal(one, whole)
    # world shard models on this device
    shards = [D.Model(cfg, b.wd, max_pos_for(cfg, b.cap), vocab_range=r)
              for r in VP.shard_bounds(cfg.V, world)]
    wss = [m.workspace(cfg.batch, cfg.B, 0) for m in shards]
    try:
        res = _emulated_draft(shards, wss, anchors, ctx, kc, vc, cfg.B, cfg.steps, cfg.batch)
    finally:
        for m in shards:
            m.close()
    for out, cst in res:
        assert torch.equal(out, res[0][0]) and torch.equal(cst, res[0][1])
    assert torch.equal(res[0][0], whole.cpu()) and torch.equal(res[0][1], wcst.cpu())
    # and the oracle's draft rules for a few requests
    rep = DraftReport()
    ctx_h = ctx.cpu()
    for r in range(min(cfg.batch, 3)):
        T = int(ctx_h[r])
        caches = oracle_caches_from(kc, vc, cfg.L, r, T)
        check_draft_request(b, r, int(anchors[r]), T, caches, res[0][0][r], res[0][1][r], None,
                            cfg.steps, rep)
    rep.save(f"vocab_parallel_draft[{name},world{world}]", config=cfg.name)


def test_shard_model_refuses_the_one_call_draft():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=2, ctx=("fixed", 64), I=512, d=512,
                 H_t=512).replace(name="vp_refuse")
    b = built(cfg)
    m = D.Model(cfg, b.wd, max_pos_for(cfg, b.cap), vocab_range=(0, 1024))
    try:
        kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
        out = torch.zeros((2, cfg.B), dtype=torch.int32, device="cuda")
        with pytest.raises(D.DFlashError) as e:
            D.draft_block(m, torch.tensor([1, 2], dtype=torch.int32).cuda(),
                          torch.tensor([64, 64], dtype=torch.int32).cuda(), kc.cuda(), vc.cuda(),
                          cfg.B, cfg.steps, out, m.workspace(2, cfg.B, 0))
        assert e.value.status == D.EUNSUPPORTED
    finally:
        m.close()
