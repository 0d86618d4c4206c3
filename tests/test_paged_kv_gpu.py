"""Paged K/V with prefix sharing on the GPU (oracle/paged_kv.py).

* Injection through a random page permutation writes, at every mapped
  position, exactly what contiguous injection writes (same arithmetic, other
  addresses), agrees with the oracle's paged injection within 1e-2 of
  max |oracle|, and leaves spare pages untouched.
* Drafting through the table gives bit for bit the contiguous draft (tokens,
  commit steps, logits) and passes the oracle's draft rules on the gathered
  context.
* A request that shares another's prefix pages and injects only its own
  suffix drafts as the oracle drafts with its whole context.
* Unmapped pages: the request writes nothing and DFLASH_DEV_PAGE is set.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth.configs import shrink
from tests.gpu_common import (DraftReport, built, check_draft_request, rel_err, REL_TOL)
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu

PK = O.paged_kv
SENTINEL = 1234.0


def _small(batch=4, ctx=("uniform", 40, 600), B=8, steps=2, name="paged8b"):
    base = synth.get_config("qwen3_8b_bs32")
    return shrink(base, L=2, V=4096, batch=batch, ctx=ctx, I=1024, d=1024, H_t=512).replace(
        B=B, steps=steps, name=name)


def _pools(cfg, n_pages, page, dtype):
    shp = (cfg.L, n_pages, cfg.nkv, page, cfg.hd)
    return (torch.full(shp, SENTINEL, dtype=dtype, device="cuda"),
            torch.full(shp, SENTINEL, dtype=dtype, device="cuda"))


def _perm_table(batch, max_pages, n_pages, seed):
    g = torch.Generator().manual_seed(seed)
    ids = torch.randperm(n_pages, generator=g)[:batch * max_pages]
    return ids.view(batch, max_pages).to(torch.int32)


def _gather(pool, table, r, T, page):
    """[L, nkv, T, hd] of request r's first T positions, read through its table."""
    pos = torch.arange(T)
    pages = table[r, pos // page].long().to(pool.device)
    slots = (pos % page).to(pool.device)
    by_slot = pool.permute(1, 3, 0, 2, 4)  # [n_pages, page, L, nkv, hd]
    return by_slot[pages, slots].permute(1, 2, 0, 3)


def test_paged_injection_and_draft_match_contiguous_and_oracle():
    cfg = _small()
    b = built(cfg)
    page = 64
    ctx = synth.make_ctx_lens(cfg)
    max_pages = -(-b.cap // page)
    n_pages = cfg.batch * max_pages + 7  # spare pages stay untouched
    # the paged draft sizes its split-KV chunks from max_pages * page + B (bounded
    # by the RoPE table); a contiguous cache of that capacity gets the same chunks
    cap = min(max_pages * page + cfg.B, b.model.max_pos)
    table = _perm_table(cfg.batch, max_pages, n_pages, 5)
    cu, st, n = synth.make_inject_layout(cfg, ctx, "prefill")
    taps = synth.make_tap_hiddens(cfg, n, label="paged_taps")
    dt = [t.cuda() for t in taps]
    kc = torch.zeros((cfg.L, cfg.batch, cfg.nkv, cap, cfg.hd), dtype=b.model.cache_dtype,
                     device="cuda")
    vc = torch.zeros_like(kc)
    kp, vp = _pools(cfg, n_pages, page, b.model.cache_dtype)
    ws = b.model.workspace(cfg.batch, cfg.B, n)
    D.inject_kv(b.model, dt, cu.cuda(), st.cuda(), kc, vc, ws)
    D.inject_kv_paged(b.model, dt, cu.cuda(), st.cuda(), kp, vp, table.cuda(), ws)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    for r in range(cfg.batch):
        T = int(ctx[r])
        assert torch.equal(_gather(kp, table, r, T, page), kc[:, r, :, :T])
        assert torch.equal(_gather(vp, table, r, T, page), vc[:, r, :, :T])
    used = set(table.flatten().tolist())
    spare = [p for p in range(n_pages) if p not in used]
    assert (kp[:, spare] == SENTINEL).all() and (vp[:, spare] == SENTINEL).all()
    # the oracle's paged injection, on the mapped positions of every request
    Kp0 = np.zeros((cfg.L, n_pages, cfg.nkv, page, cfg.hd))
    Kpo, Vpo, status = PK.inject_kv_paged(taps, cu, st, table.numpy(), page, b.W, cfg, Kp0, Kp0)
    assert (status == PK.STATUS_OK).all()
    worst = 0.0
    for r in range(cfg.batch):
        T = int(ctx[r])
        Ko = PK.gather_caches(Kpo, Vpo, table[r].numpy(), T, page)
        for l in range(cfg.L):
            gk = _gather(kp, table, r, T, page)[l].float().cpu().numpy().transpose(1, 0, 2)
            gv = _gather(vp, table, r, T, page)[l].float().cpu().numpy().transpose(1, 0, 2)
            e = max(rel_err(gk, Ko[l][0]), rel_err(gv, Ko[l][1]))
            worst = max(worst, e)
            assert e <= REL_TOL, (r, l, e)

    # drafting through the table: bit for bit the contiguous draft
    anchors = synth.make_anchors(cfg)
    outs = []
    for paged in (False, True):
        out = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
        cst = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
        lg = torch.full((cfg.steps, cfg.batch, cfg.B, cfg.V), float("nan"), device="cuda")
        wsd = b.model.workspace(cfg.batch, cfg.B, 0)
        if paged:
            D.draft_block_paged(b.model, anchors.cuda(), ctx.cuda(), kp, vp, table.cuda(), cfg.B,
                                cfg.steps, out, wsd, commit_step=cst, logits_dbg=lg)
        else:
            D.draft_block(b.model, anchors.cuda(), ctx.cuda(), kc, vc, cfg.B, cfg.steps, out, wsd,
                          commit_step=cst, logits_dbg=lg)
        torch.cuda.synchronize()
        assert D.get_error(wsd) == 0
        outs.append((out.cpu(), cst.cpu(), lg))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(torch.nan_to_num(outs[0][2], 9.0), torch.nan_to_num(outs[1][2], 9.0))
    # and the oracle's paged draft rules, on the context gathered through the table
    rep = DraftReport()
    out, cst, lg = outs[1]
    for r in range(cfg.batch):
        T = int(ctx[r])
        caches = PK.gather_caches(O.as_f64(kp), O.as_f64(vp), table[r].numpy(), T, page)
        glog = [{p: lg[t, r, p].cpu().numpy() for p in range(1, cfg.B)} for t in range(cfg.steps)]
        check_draft_request(b, r, int(anchors[r]), T, caches, out[r], cst[r], glog, cfg.steps, rep)
    rep.save("paged_draft_vs_oracle", config=cfg.name, max_kv_rel=worst)
    print(rep, worst)


def test_paged_prefix_sharing():
    """Request 1 shares request 0's first `shared` positions (whole pages, the same
    tapped states) and injects only its own suffix into pages of its own.  Its
    draft equals the oracle's draft of request 1 with the whole context private."""
    cfg = _small(batch=2, ctx=("fixed", 320), name="share8b")
    b = built(cfg)
    page, shared = 64, 192
    T = 320
    max_pages = 6
    # request 0: pages 0..4; request 1: shares pages 0..2, then its own pages 5, 6
    table = torch.tensor([[0, 1, 2, 3, 4, -1], [0, 1, 2, 5, 6, -1]], dtype=torch.int32)
    n_pages = 8
    taps0 = synth.make_tap_hiddens(cfg, T, label="share_req0")
    tail1 = synth.make_tap_hiddens(cfg, T - shared, label="share_req1_tail")
    kp, vp = _pools(cfg, n_pages, page, b.model.cache_dtype)
    # call 1: request 0's whole context; call 2: request 1's suffix only
    ws = b.model.workspace(2, cfg.B, T)
    D.inject_kv_paged(b.model, [t.cuda() for t in taps0],
                      torch.tensor([0, T, T], dtype=torch.int32).cuda(),
                      torch.tensor([0, 0], dtype=torch.int32).cuda(), kp, vp, table.cuda(), ws)
    D.inject_kv_paged(b.model, [t.cuda() for t in tail1],
                      torch.tensor([0, 0, T - shared], dtype=torch.int32).cuda(),
                      torch.tensor([0, shared], dtype=torch.int32).cuda(), kp, vp, table.cuda(), ws)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    assert (kp[:, 7] == SENTINEL).all()
    anchors = torch.tensor([11, 12], dtype=torch.int32)
    ctx = torch.tensor([T, T], dtype=torch.int32)
    out = torch.full((2, cfg.B), -5, dtype=torch.int32, device="cuda")
    cst = torch.full((2, cfg.B), -5, dtype=torch.int32, device="cuda")
    lg = torch.full((cfg.steps, 2, cfg.B, cfg.V), float("nan"), device="cuda")
    wsd = b.model.workspace(2, cfg.B, 0)
    D.draft_block_paged(b.model, anchors.cuda(), ctx.cuda(), kp, vp, table.cuda(), cfg.B,
                        cfg.steps, out, wsd, commit_step=cst, logits_dbg=lg)
    torch.cuda.synchronize()
    assert D.get_error(wsd) == 0
    # the oracle: request 1's whole context injected privately (its prefix taps are
    # request 0's), then drafted
    full1 = [torch.cat([a[:shared], t]) for a, t in zip(taps0, tail1)]
    inj = O.inject_kv_requests(full1, torch.tensor([0, T]), torch.tensor([0]), b.W, cfg)
    caches = [(inj[(l, 0)][1], inj[(l, 0)][2]) for l in range(cfg.L)]
    rep = DraftReport()
    glog = [{p: lg[t, 1, p].cpu().numpy() for p in range(1, cfg.B)} for t in range(cfg.steps)]
    check_draft_request(b, 1, 12, T, caches, out[1].cpu(), cst[1].cpu(), glog, cfg.steps, rep)
    rep.save("paged_prefix_sharing", config=cfg.name)
    print(rep)


def test_paged_unmapped_pages_write_nothing():
    cfg = _small(batch=3, ctx=("fixed", 200), name="unmapped8b")
    b = built(cfg)
    page, T, max_pages, n_pages = 64, 192, 4, 12
    table = torch.tensor([[0, 1, 2, 3], [4, -1, 6, 7], [8, 9, 10, 99]], dtype=torch.int32)
    taps = [t.cuda() for t in synth.make_tap_hiddens(cfg, 3 * T, label="unmapped")]
    kp, vp = _pools(cfg, n_pages, page, b.model.cache_dtype)
    ws = b.model.workspace(3, cfg.B, 3 * T)
    cu = torch.tensor([0, T, 2 * T, 3 * T], dtype=torch.int32).cuda()
    D.inject_kv_paged(b.model, taps, cu, torch.zeros(3, dtype=torch.int32).cuda(), kp, vp,
                      table.cuda(), ws)
    torch.cuda.synchronize()
    # request 1 touches table entry 1 (-1): nothing written; request 2's 192
    # positions fill pages 8..10, so its out-of-pool last entry is never touched
    assert D.get_error(ws) == D.DEV_PAGE
    assert (kp[:, [4, 6, 7]] == SENTINEL).all()
    assert (kp[:, [0, 1, 2]] != SENTINEL).all() and (kp[:, [8, 9, 10]] != SENTINEL).all()
    # drafting: request 1 has an unmapped page below its context
    out = torch.full((3, cfg.B), -5, dtype=torch.int32, device="cuda")
    wsd = b.model.workspace(3, cfg.B, 0)
    D.draft_block_paged(b.model, torch.tensor([1, 2, 3], dtype=torch.int32).cuda(),
                        torch.full((3,), T, dtype=torch.int32).cuda(), kp, vp, table.cuda(),
                        cfg.B, cfg.steps, out, wsd)
    torch.cuda.synchronize()
    assert D.get_error(wsd) == D.DEV_PAGE
    o = out.cpu()
    assert (o[1] == -5).all() and (o[0] >= 0).all() and (o[2] >= 0).all()


def test_paged_draft_full_size_matches_contiguous():
    """The 8B-shaped batch of 32 (contexts up to 4096) with 256-position pages in a
    shuffled pool: the paged draft is the contiguous draft, bit for bit."""
    cfg = synth.get_config("qwen3_8b_bs32")
    b = built(cfg)
    page = 256
    max_pages = -(-b.cap // page)
    n_pages = cfg.batch * max_pages
    cap = min(max_pages * page + cfg.B, b.model.max_pos)  # same split-KV chunks as paged
    table = _perm_table(cfg.batch, max_pages, n_pages, 9)
    kc, vc = synth.make_kv_cache(cfg, cap, dtype=b.model.cache_dtype)
    kc, vc = kc.cuda(), vc.cuda()
    kp, vp = _pools(cfg, n_pages, page, b.model.cache_dtype)
    # scatter the contiguous cache into the pool through the table
    for r in range(cfg.batch):
        for k in range(max_pages):
            lo, hi = k * page, min(cap, (k + 1) * page)
            if hi > lo:
                kp[:, int(table[r, k]), :, :hi - lo] = kc[:, r, :, lo:hi]
                vp[:, int(table[r, k]), :, :hi - lo] = vc[:, r, :, lo:hi]
    ctx = synth.make_ctx_lens(cfg)
    anchors = synth.make_anchors(cfg).cuda()
    res = []
    for paged in (False, True):
        out = torch.zeros((cfg.batch, cfg.B), dtype=torch.int32, device="cuda")
        cst = torch.zeros((cfg.batch, cfg.B), dtype=torch.int32, device="cuda")
        wsd = b.model.workspace(cfg.batch, cfg.B, 0)
        if paged:
            D.draft_block_paged(b.model, anchors, ctx.cuda(), kp, vp, table.cuda(), cfg.B,
                                cfg.steps, out, wsd, commit_step=cst)
        else:
            D.draft_block(b.model, anchors, ctx.cuda(), kc, vc, cfg.B, cfg.steps, out, wsd,
                          commit_step=cst)
        torch.cuda.synchronize()
        assert D.get_error(wsd) == 0
        res.append((out.cpu(), cst.cpu()))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
