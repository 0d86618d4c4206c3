"""Masked-block draft forward on the GPU against the oracle.

The K/V cache is filled with seeded synthetic values (the injection path has
its own tests), so the oracle can recompute any request from the same cache.
Draft tokens must equal the oracle's argmax except at near-ties (top-2 margin
< 0.05); LM-head logits of every masked row agree within 1e-2 of max |oracle|;
commit sets must be admitted by the oracle (see tests/gpu_common.py).
"""

import pytest
import torch

import oracle as O
import synth
from synth.configs import shrink
from tests.gpu_common import DraftReport, built, check_draft_request, oracle_caches_from, record
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def _run_draft(b, cfg, steps=None, dbg=True, ctx=None, anchors=None):
    steps = cfg.steps if steps is None else steps
    ctx = synth.make_ctx_lens(cfg) if ctx is None else ctx
    anchors = synth.make_anchors(cfg) if anchors is None else anchors
    kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
    dk, dv = kc.cuda(), vc.cuda()
    out = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
    cst = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
    lg = (torch.full((steps, cfg.batch, cfg.B, cfg.V), float("nan"), device="cuda")
          if dbg else None)
    ws = b.model.workspace(cfg.batch, cfg.B, 0)
    D.draft_block(b.model, anchors.cuda(), ctx.cuda(), dk, dv, cfg.B, steps, out, ws,
                  commit_step=cst, logits_dbg=lg)
    torch.cuda.synchronize()
    return dict(ctx=ctx, anchors=anchors, kc=kc, vc=vc, out=out.cpu(), cst=cst.cpu(),
                lg=lg, err=D.get_error(ws))


def _check(b, cfg, res, steps, requests, test=None):
    rep = DraftReport()
    for r in requests:
        T = int(res["ctx"][r])
        caches = oracle_caches_from(res["kc"], res["vc"], cfg.L, r, T)
        glog = None
        if res["lg"] is not None:
            glog = [{p: res["lg"][t, r, p].cpu().numpy() for p in range(1, cfg.B)}
                    for t in range(steps)]
        check_draft_request(b, r, int(res["anchors"][r]), T, caches, res["out"][r],
                            res["cst"][r], glog, steps, rep)
        assert int(res["cst"][r][0]) == -1
    if test:
        rep.save(test, config=cfg.name, requests=len(list(requests)))
    return rep


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_draft_tiny(dtype):
    cfg = synth.get_config("tiny_f32", dtype=dtype, name=f"tiny_{dtype}")
    b = built(cfg)
    res = _run_draft(b, cfg)
    assert res["err"] == 0
    rep = _check(b, cfg, res, cfg.steps, range(cfg.batch), test=f"draft_tiny[{dtype}]")
    if dtype == "f32":
        assert rep.max_logit_rel < 1e-5 and rep.token_near_ties == 0
    print(rep)


@pytest.mark.parametrize("steps", [1, 2, 3])
def test_draft_tiny_bf16_denoising_steps(steps):
    cfg = synth.get_config("tiny_f32", dtype="bf16", name="tiny_bf16", batch=3)
    b = built(cfg)
    res = _run_draft(b, cfg, steps=steps)
    assert res["err"] == 0
    print(_check(b, cfg, res, steps, range(cfg.batch), test=f"draft_tiny_bf16_steps[{steps}]"))


@pytest.mark.parametrize("B,steps", [(8, 2), (16, 1), (4, 3)])
def test_draft_small_8b_geometry(B, steps):
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=4096, batch=5, ctx=("uniform", 30, 700), I=1024, d=1024,
                 H_t=512).replace(B=B, steps=steps, name=f"small8b_B{B}")
    b = built(cfg)
    res = _run_draft(b, cfg)
    assert res["err"] == 0
    print(_check(b, cfg, res, steps, range(cfg.batch), test=f"draft_small_8b[B{B},s{steps}]"))


def test_draft_context_lengths_edge_cases():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=4, ctx=("fixed", 600), I=512, d=512, H_t=512).replace(
        name="edge8b")
    b = built(cfg)
    # empty context, one position, a full chunk boundary, the longest context the cache holds
    ctx = torch.tensor([0, 1, 256, b.cap - cfg.B], dtype=torch.int32)
    res = _run_draft(b, cfg, ctx=ctx)
    assert res["err"] == 0
    print(_check(b, cfg, res, cfg.steps, range(cfg.batch), test="draft_context_edge_cases"))


@pytest.mark.parametrize("sched", [0, 2])
@pytest.mark.parametrize("chunk", [64, 192, 4096])
def test_draft_attention_chunk_sizes(chunk, sched):
    """The same requests with the split-KV chunk forced from one tile per chunk to one
    chunk per request: every split and the chunk combine give the oracle's result, on
    the mma.sync kernel (schedule 0) and on the tcgen05 kernel (schedule 2)."""
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=4, ctx=("uniform", 1, 900), I=512, d=512,
                 H_t=512).replace(name="chunk8b")
    b = built(cfg)
    ctx = torch.tensor([0, 63, 64, 900], dtype=torch.int32)
    D.debug_attn_chunk(chunk)  # the split-KV grid
    D.debug_attn_schedule(sched)
    try:
        res = _run_draft(b, cfg, ctx=ctx)
    finally:
        D.debug_attn_chunk(0)
        D.debug_attn_schedule(0)
    assert res["err"] == 0
    print(chunk, sched, _check(b, cfg, res, cfg.steps, range(cfg.batch),
                               test=f"draft_attention_chunk[{chunk}-{sched}]"))


def test_draft_rejects_bad_requests_without_writing():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=3, ctx=("fixed", 16), I=512, d=512, H_t=512).replace(
        name="bad8b")
    b = built(cfg)
    ctx = torch.tensor([16, b.cap - cfg.B + 1, 16], dtype=torch.int32)  # request 1 overflows
    anchors = torch.tensor([5, 6, cfg.V], dtype=torch.int32)            # request 2 out of range
    res = _run_draft(b, cfg, ctx=ctx, anchors=anchors, dbg=False)
    assert res["err"] == D.DEV_CTX_CAP | D.DEV_TOKEN_RANGE
    assert (res["out"][1] == -5).all() and (res["out"][2] == -5).all()
    assert int(res["out"][0][0]) == 5 and (res["out"][0] >= 0).all()


@pytest.mark.parametrize("name,requests", [
    ("qwen3_4b_bs1", [0]),
    ("qwen3_8b_bs32", [0, 13, 31]),
    ("qwen3_8b_ctx32k", [2]),
])
def test_draft_full_size_sampled_requests(name, requests):
    cfg = synth.get_config(name)
    b = built(cfg)
    res = _run_draft(b, cfg)
    assert res["err"] == 0
    # every request produced a complete block
    out = res["out"]
    assert (out[:, 1:] >= 0).all() and (out[:, 1:] < cfg.V).all()
    assert (res["cst"][:, 1:] >= 0).all() and (res["cst"][:, 1:] < cfg.steps).all()
    print(name, _check(b, cfg, res, cfg.steps, requests, test=f"draft_full_size[{name}]"))


@pytest.mark.parametrize("name,requests", [
    ("qwen3_8b_bs32", [5]),
    ("qwen3_8b_ctx32k", [1]),   # 43 split-KV chunks per request: a long chunk merge
])
def test_draft_full_size_tcgen05_attention(name, requests):
    """At full size the split-KV grid on the tcgen05 kernel gives a draft that
    passes the oracle's rules on the sampled requests, and logits that agree with
    the default mma.sync kernel far inside the tolerance (every denoising step
    where both committed the same tokens, else the first)."""
    cfg = synth.get_config(name)
    b = built(cfg)
    base = _run_draft(b, cfg)
    try:
        D.debug_attn_schedule(2)
        umma = _run_draft(b, cfg)
    finally:
        D.debug_attn_schedule(0)
    assert base["err"] == 0 and umma["err"] == 0
    _check(b, cfg, umma, cfg.steps, requests, test=f"draft_full_size_tcgen05_attention[{name}]")
    same = torch.equal(base["out"], umma["out"]) and torch.equal(base["cst"], umma["cst"])
    la, lb = base["lg"], umma["lg"]
    if not same:
        la, lb = la[:1], lb[:1]
    both = ~(torch.isnan(la) | torch.isnan(lb))
    scale = la[both].abs().max().item()
    diff = (la[both] - lb[both]).abs().max().item()
    record("draft_full_size_tcgen05_attention", max_rel_diff=diff / scale, configs=1,
           configs_same_commits=int(same))
    assert diff <= 2e-3 * scale


def test_draft_gemm_schedules_agree():
    """The GEMM schedules (the default: stream-K LM head and fixed-split
    projections; fixed splits everywhere; stream-K everywhere, every split tile
    finished inside the GEMM with the fused epilogues) compute the same products
    up to fp32 summation order: every draft passes the oracle's rules, and their
    logits agree far inside the tolerance."""
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=4096, batch=5, ctx=("uniform", 30, 700), I=1024, d=1024,
                 H_t=512).replace(name="small8b_B8")
    b = built(cfg)
    runs = []
    try:
        for sched in (0, 1, 2):
            D.debug_gemm_schedule(sched)
            runs.append(_run_draft(b, cfg))
    finally:
        D.debug_gemm_schedule(0)
    for res in runs:
        assert res["err"] == 0
        _check(b, cfg, res, cfg.steps, range(cfg.batch))
    la = runs[0]["lg"]
    for other in runs[1:]:
        lb = other["lg"]
        both = ~(torch.isnan(la) | torch.isnan(lb))
        scale = la[both].abs().max().item()
        diff = (la[both] - lb[both]).abs().max().item()
        record("draft_gemm_schedules", max_rel_diff=diff / scale)
        assert diff <= 2e-3 * scale


@pytest.mark.parametrize("name,ctx", [
    ("edge", (0, 1, 63, 64, 65, 600)),   # empty, one key, tile edges, a long one
    ("uniform", None),
])
def test_draft_attention_schedules_agree(name, ctx):
    """The three attention schedules give the oracle's draft, and their logits
    agree far inside the tolerance: the persistent mma.sync attention (every CTA
    the same number of key tiles across (request, head) segments, segments split
    between CTAs merged by their last piece), the split-KV grid on the mma.sync
    kernel (the default) and the split-KV grid on the tcgen05 kernel."""
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=2048, batch=6, ctx=("uniform", 1, 700), I=512, d=512,
                 H_t=512).replace(name="attn_sched8b")
    b = built(cfg)
    ctx_t = None if ctx is None else torch.tensor(ctx, dtype=torch.int32)
    runs = []
    try:
        for sched in (1, 0, 2):
            D.debug_attn_schedule(sched)
            runs.append(_run_draft(b, cfg, ctx=ctx_t))
    finally:
        D.debug_attn_schedule(0)
    for res in runs:
        assert res["err"] == 0
        _check(b, cfg, res, cfg.steps, range(cfg.batch), test=f"draft_attention_schedules[{name}]")
    # the first denoising step depends on no commit decision; later steps are
    # compared where both schedules committed the same tokens (each run's
    # near-tie choices are checked against the oracle's rules above)
    for other in runs[1:]:
        same = torch.equal(runs[0]["out"], other["out"]) and torch.equal(runs[0]["cst"],
                                                                            other["cst"])
        la, lb = runs[0]["lg"], other["lg"]
        if not same:
            la, lb = la[:1], lb[:1]
        both = ~(torch.isnan(la) | torch.isnan(lb))
        scale = la[both].abs().max().item()
        assert (la[both] - lb[both]).abs().max().item() <= 2e-3 * scale
