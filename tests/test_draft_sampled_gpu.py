"""Sampled (temperature) drafting on the GPU against the oracle
(oracle/sampled_draft.py).

Both sides draw with the same Philox4x64-10 noise (stream 2), so every draw
has one right answer for given logits.  The GPU's logits differ from the
oracle's fp64 logits within the draft tolerance, so the checks are, for each
request and denoising step (the oracle walks the steps, teacher-forced to
the GPU's admitted choices as in the greedy tests):

* the committed position's stored logits row (the q row sampled verify takes)
  is within 1e-2 of max |oracle| of the oracle's logits of that step;
* the draw is exact on the stored row: recomputing argmax(q / tau + G) in
  float64 from the row the GPU returned gives the GPU's token, unless the two
  best scores are within fp32 rounding (counted);
* the token is the oracle's draw, or one whose oracle score is within
  0.05 / tau of the oracle's best (a logit near-tie scaled by the temperature;
  counted);
* the commit set is admitted: every committed position's confidence (the
  untempered probability of its token under the oracle's logits) is at least
  (1 - 0.05) times the confidence of every excluded position, taking for each
  excluded position the least confident token its near-tie band admits.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth.configs import shrink
from tests.gpu_common import (DraftReport, built, check_draft_request, oracle_caches_from,
                              rel_err, REL_TOL)
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu

SD = O.sampled_draft
SV = O.sampled_verify
SEED, OFFSET = 0x5EED, 7
SCORE_BAND = 0.05     # logit near-tie band, divided by the temperature for scores
CONF_BAND = 0.05
FP32_SCORE_TIE = 1e-5


class SampledReport(DraftReport):
    def __init__(self):
        super().__init__()
        self.draw_fp32_ties = 0

    def save(self, test, **extra):
        return super().save(test, draw_fp32_ties=self.draw_fp32_ties, **extra)


def _gumbel(r, t, p, B, V):
    return -np.log(SD.draft_draw_exponentials(SEED, OFFSET, r, t, p, B, V))


def check_sampled_request(b, r, anchor, T, caches, tokens_gpu, cstep_gpu, q_gpu, steps, tau,
                          rep):
    cfg = b.cfg
    B, V = cfg.B, cfg.V
    tokens = np.full(B, cfg.mask_id, dtype=np.int64)
    tokens[0] = anchor
    assert int(tokens_gpu[0]) == anchor
    masked = list(range(1, B))
    for t in range(steps):
        z = O.draft_hidden(tokens, T, caches, b.W, cfg)
        Y = b.W.lm_logits(z[masked])
        k = O.commit_count(len(masked), steps - t)
        commit = sorted(p for p in masked if int(cstep_gpu[p]) == t)
        assert len(commit) == k, (r, t, commit, k)
        conf_in, conf_out_lo = [], []
        for i, p in enumerate(masked):
            G = _gumbel(r, t, p, B, V)
            S = Y[i] / tau + G
            x_o = int(np.argmax(S))
            lp1 = SV.log_softmax(Y[i], 1.0)
            admit = np.nonzero(S >= S[x_o] - SCORE_BAND / tau)[0]
            if p in commit:
                g = int(tokens_gpu[p])
                q = q_gpu[p]
                e = rel_err(q, Y[i])
                rep.max_logit_rel = max(rep.max_logit_rel, e)
                assert e <= REL_TOL, f"req {r} step {t} pos {p}: q row rel err {e:.3e}"
                Sq = q / tau + G
                x_q = int(np.argmax(Sq))
                if g != x_q:
                    assert Sq[x_q] - Sq[g] <= FP32_SCORE_TIE * max(1.0, abs(Sq[x_q])), (
                        f"req {r} step {t} pos {p}: drew {g}, its own row gives {x_q}")
                    rep.draw_fp32_ties += 1
                rep.positions += 1
                if g != x_o:
                    assert g in set(int(v) for v in admit), (
                        f"req {r} step {t} pos {p}: drew {g}, oracle {x_o} "
                        f"(score gap {S[x_o] - S[g]:.4f})")
                    rep.token_near_ties += 1
                conf_in.append(float(np.exp(lp1[g])))
                tokens[p] = g
            else:
                conf_out_lo.append(float(np.exp(lp1[admit]).min()))
        if conf_out_lo:
            worst_in, best_out = min(conf_in), max(conf_out_lo)
            if worst_in < best_out:
                assert worst_in >= (1.0 - CONF_BAND) * best_out, (
                    f"req {r} step {t}: commit {commit} not admitted "
                    f"({worst_in:.6f} < {best_out:.6f})")
                rep.commit_near_ties += 1
        masked = [p for p in masked if p not in commit]
    assert not masked


def _run(b, cfg, tau, steps, q_dtype, ctx=None, anchors=None, kv=None):
    ctx = synth.make_ctx_lens(cfg) if ctx is None else ctx
    anchors = synth.make_anchors(cfg) if anchors is None else anchors
    kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype) if kv is None else kv
    dk, dv = kc.cuda(), vc.cuda()
    out = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
    cst = torch.full((cfg.batch, cfg.B), -5, dtype=torch.int32, device="cuda")
    q = torch.full((cfg.batch, cfg.B, cfg.V), -7.0, dtype=q_dtype, device="cuda")
    ws = b.model.workspace(cfg.batch, cfg.B, 0)
    D.draft_block_sampled(b.model, anchors.cuda(), ctx.cuda(), dk, dv, cfg.B, steps, tau, SEED,
                          OFFSET, out, q, ws, commit_step=cst)
    torch.cuda.synchronize()
    return dict(ctx=ctx, anchors=anchors, kc=kc, vc=vc, out=out.cpu(), cst=cst.cpu(),
                q=q.double().cpu().numpy(), err=D.get_error(ws))


def _check_all(b, cfg, res, tau, steps, requests, test):
    rep = SampledReport()
    for r in requests:
        T = int(res["ctx"][r])
        caches = oracle_caches_from(res["kc"], res["vc"], cfg.L, r, T)
        check_sampled_request(b, r, int(res["anchors"][r]), T, caches, res["out"][r],
                              res["cst"][r], res["q"][r], steps, tau, rep)
        assert int(res["cst"][r][0]) == -1
        assert (res["q"][r][0] == -7.0).all()  # row 0 (the anchor) is not written
    rep.save(test, config=cfg.name, tau=tau, steps=steps, requests=len(list(requests)))
    print(test, rep, "fp32 draw ties", rep.draw_fp32_ties)
    return rep


@pytest.mark.parametrize("dtype,tau,steps", [("f32", 1.0, 1), ("f32", 0.7, 3), ("bf16", 1.5, 2),
                                             ("bf16", 1.0, 1)])
def test_sampled_draft_tiny(dtype, tau, steps):
    cfg = synth.get_config("tiny_f32", dtype=dtype, name=f"tiny_{dtype}", batch=3)
    b = built(cfg)
    q_dtype = torch.float32 if dtype == "f32" else torch.bfloat16
    res = _run(b, cfg, tau, steps, q_dtype)
    assert res["err"] == 0
    _check_all(b, cfg, res, tau, steps, range(cfg.batch),
               f"sampled_draft_tiny[{dtype},tau{tau},s{steps}]")


@pytest.mark.parametrize("B,steps,q_dtype", [(8, 2, torch.bfloat16), (16, 1, torch.float32),
                                             (4, 3, torch.float32)])
def test_sampled_draft_small_8b_geometry(B, steps, q_dtype):
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=4096, batch=5, ctx=("uniform", 30, 700), I=1024, d=1024,
                 H_t=512).replace(B=B, steps=steps, name=f"small8b_B{B}")
    b = built(cfg)
    res = _run(b, cfg, 1.0, steps, q_dtype)
    assert res["err"] == 0
    _check_all(b, cfg, res, 1.0, steps, range(cfg.batch), f"sampled_draft_small_8b[B{B},s{steps}]")


def test_sampled_draft_full_size_sampled_requests():
    cfg = synth.get_config("qwen3_8b_bs32")
    b = built(cfg)
    res = _run(b, cfg, 1.0, cfg.steps, torch.bfloat16)
    assert res["err"] == 0
    out = res["out"]
    assert (out[:, 1:] >= 0).all() and (out[:, 1:] < cfg.V).all()
    assert (res["cst"][:, 1:] >= 0).all() and (res["cst"][:, 1:] < cfg.steps).all()
    _check_all(b, cfg, res, 1.0, cfg.steps, [0, 13, 31], "sampled_draft_full_size[qwen3_8b_bs32]")


def test_sampled_draft_low_temperature_is_the_greedy_draft():
    """At temperature 1e-4 the draw is the argmax (the Gumbel noise moves scores by
    less than 1e-2 logits) and the confidence the max-probability: the greedy
    checks hold for the sampled call."""
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=4096, batch=5, ctx=("uniform", 30, 700), I=1024, d=1024,
                 H_t=512).replace(name="small8b_B8")
    b = built(cfg)
    res = _run(b, cfg, 1e-4, cfg.steps, torch.float32)
    assert res["err"] == 0
    rep = DraftReport()
    for r in range(cfg.batch):
        T = int(res["ctx"][r])
        caches = oracle_caches_from(res["kc"], res["vc"], cfg.L, r, T)
        check_draft_request(b, r, int(res["anchors"][r]), T, caches, res["out"][r],
                            res["cst"][r], None, cfg.steps, rep)
    rep.save("sampled_draft_tau_1e-4_vs_greedy", config=cfg.name)


def test_sampled_draft_repeats_with_equal_seed_and_offset():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=4, ctx=("uniform", 30, 300), I=512, d=512,
                 H_t=512).replace(name="rep8b")
    b = built(cfg)
    r1 = _run(b, cfg, 1.3, cfg.steps, torch.float32)
    r2 = _run(b, cfg, 1.3, cfg.steps, torch.float32)
    assert np.array_equal(r1["out"], r2["out"]) and np.array_equal(r1["q"], r2["q"])


def test_sampled_draft_bad_requests_write_nothing():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=3, ctx=("fixed", 16), I=512, d=512, H_t=512).replace(
        name="bad8b")
    b = built(cfg)
    ctx = torch.tensor([16, b.cap - cfg.B + 1, 16], dtype=torch.int32)  # request 1 overflows
    anchors = torch.tensor([5, 6, cfg.V], dtype=torch.int32)            # request 2 out of range
    res = _run(b, cfg, 1.0, cfg.steps, torch.float32, ctx=ctx, anchors=anchors)
    assert res["err"] == D.DEV_CTX_CAP | D.DEV_TOKEN_RANGE
    for r in (1, 2):
        assert (res["out"][r] == -5).all() and (res["cst"][r] == -5).all()
        assert (res["q"][r] == -7.0).all()
    assert int(res["out"][0][0]) == 5 and (res["out"][0] >= 0).all()
    assert (res["q"][0][1:] != -7.0).any(axis=1).all()


def test_sampled_draft_then_sampled_verify_accepts_a_matching_target():
    """Drafting, then sampled verify against a target whose row i is the draft's
    own distribution for position i + 1: every ratio p/q is 1, so every request
    accepts the whole block (a = B - 1).  The verify outputs match the oracle's
    sampled verify on the same inputs."""
    from tests.test_verify_sampled_gpu import _check as sv_check

    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=4, ctx=("uniform", 30, 300), I=512, d=512,
                 H_t=512).replace(name="chain_sampled8b")
    b = built(cfg)
    tau = 0.9
    res = _run(b, cfg, tau, cfg.steps, torch.float32)
    assert res["err"] == 0
    q = torch.as_tensor(res["q"], dtype=torch.float32)
    Z = torch.zeros_like(q)
    Z[:, :-1] = q[:, 1:]
    Z[:, -1] = torch.randn(cfg.batch, cfg.V, generator=torch.Generator().manual_seed(3))
    d = res["out"].to(torch.int32)
    cap = 2 * cfg.B
    out0 = torch.full((cfg.batch, cap), -1, dtype=torch.int32)
    ol0 = torch.zeros(cfg.batch, dtype=torch.int32)
    seq0 = res["ctx"].clone()
    g = {k: v.cuda() for k, v in dict(Z=Z, Y=q, d=d, out=out0, ol=ol0, seq=seq0).items()}
    acc = torch.full((cfg.batch,), -9, dtype=torch.int32, device="cuda")
    nxt = torch.full((cfg.batch,), -9, dtype=torch.int32, device="cuda")
    ws = D.new_workspace(D.verify_sampled_workspace_size(cfg.batch, cfg.B, cfg.V))
    D.verify_sampled(g["Z"], g["Y"], g["d"], tau, SEED, OFFSET + 1, g["out"], g["ol"], g["seq"],
                     acc, nxt, ws)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    assert (acc.cpu() == cfg.B - 1).all()
    got = {"out_tokens": g["out"].cpu().numpy(), "out_len": g["ol"].cpu().numpy(),
           "seq_lens": g["seq"].cpu().numpy(), "accept": acc.cpu().numpy(),
           "next_anchor": nxt.cpu().numpy(), "err": 0}
    stats = {"requests": 0, "accept_near_ties": 0, "draw_near_ties": 0}
    sv_check(Z, q, d, tau, SEED, OFFSET + 1, out0, ol0, seq0, got, stats)
