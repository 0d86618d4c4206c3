"""Pins for the sampled-drafting oracle (oracle/sampled_draft.py).

* tau -> 0 reproduces the greedy draft (tokens and commit sets), itself pinned
  in test_oracle_pins.py against the loop-based twin.
* With one denoising step, each position's token is a draw from
  softmax(Y_j / tau): a chi-square test over many requests.  A planted
  mistake (drawing at temperature 1) must fail it.
* Drafting followed by sampled verify against a target whose distributions
  equal the draft's accepts the whole block.
* The commit schedule: ceil(remaining / steps left) per step, every position
  committed once.  The committing step's logits are kept per position.
"""

import numpy as np
import pytest
import scipy.stats

import oracle as O
from tests.test_oracle_pins import MICRO, _micro_caches, micro_weights

SD = O.sampled_draft
SV = O.sampled_verify


def _model(B=5):
    cfg = MICRO.replace(B=B)
    W = O.Weights64(micro_weights(cfg), cfg)
    return cfg, W, _micro_caches(cfg, 3)


@pytest.mark.parametrize("steps", [1, 2, 4])
def test_zero_temperature_is_greedy_draft(steps):
    cfg, W, caches = _model(B=5)
    for anchor in (3, 7, 11):
        g_tok, g_rec = O.draft_block(anchor, 3, caches, W, cfg, steps=steps)
        s_tok, q, s_rec = SD.sampled_draft_block(anchor, 3, caches, W, cfg, 1e-5, 0x5EED, 0, 0,
                                                 steps=steps)
        np.testing.assert_array_equal(s_tok, g_tok)
        assert [r["commit"] for r in s_rec] == [r["commit"] for r in g_rec]


def _single_step_draws(n, tau, cfg, W, caches, draw_tau=None):
    """First masked position's token over n requests (one step), and its exact
    distribution softmax(Y_1 / tau) from one forward."""
    toks = np.empty(n, dtype=np.int64)
    for r in range(n):
        t, _, _ = SD.sampled_draft_block(7, 3, caches, W, cfg, draw_tau or tau, 99, 4, r,
                                         steps=1)
        toks[r] = t[1]
    z = O.draft_hidden([7] + [cfg.mask_id] * (cfg.B - 1), 3, caches, W, cfg)
    p = np.exp(SV.log_softmax(W.lm_logits(z[1:2])[0], tau))
    return toks, p


def _pooled_pvalue(toks, p, min_expected=5.0):
    """Chi-square p-value with cells of small expected count pooled into one."""
    n = len(toks)
    obs = np.bincount(toks, minlength=len(p)).astype(float)
    big = n * p >= min_expected
    o = np.append(obs[big], obs[~big].sum())
    e = np.append(n * p[big], n * p[~big].sum())
    if e[-1] == 0:
        o, e = o[:-1], e[:-1]
    return scipy.stats.chisquare(o, e).pvalue


@pytest.mark.parametrize("tau", [0.7, 1.5])
def test_single_step_draws_follow_tempered_softmax(tau):
    cfg, W, caches = _model(B=3)
    toks, p = _single_step_draws(3000, tau, cfg, W, caches)
    assert _pooled_pvalue(toks, p) > 1e-4


def test_planted_wrong_temperature_fails_the_distribution_check():
    cfg, W, caches = _model(B=3)
    toks, p = _single_step_draws(3000, 0.4, cfg, W, caches, draw_tau=1.0)
    assert _pooled_pvalue(toks, p) < 1e-8


def test_draft_then_verify_against_equal_distributions_accepts_all():
    # one step: every d_j is a draw from q_j; a target whose row i equals the
    # draft's logits at position i+1 gives p_i = q_{i+1}, so rho = 1 everywhere
    cfg, W, caches = _model(B=5)
    B, V = cfg.B, cfg.V
    for r in range(20):
        tok, q, _ = SD.sampled_draft_block(5, 3, caches, W, cfg, 0.9, 1234, 0, r, steps=1)
        Z = np.vstack([q[1:], np.random.default_rng(r).normal(size=(1, V))])
        res = SV.sampled_verify_request(Z, q, tok, 0.9, 777, 0, r)
        assert res["a"] == B - 1


def test_commit_schedule_and_committed_logits():
    cfg, W, caches = _model(B=8)
    for steps in (1, 2, 3, 7):
        tok, q, rec = SD.sampled_draft_block(2, 3, caches, W, cfg, 1.3, 5, 1, 3, steps=steps)
        rem = cfg.B - 1
        seen = []
        for t, r in enumerate(rec):
            assert len(r["commit"]) == O.commit_count(rem, steps - t)
            rem -= len(r["commit"])
            seen += r["commit"]
            for p in r["commit"]:
                i = r["pos"].index(p)
                assert tok[p] == r["draw"][i]
                np.testing.assert_array_equal(q[p], r["logits"][i])
                # committed positions are the most confident of the step
                assert all(r["conf"][i] >= c or r["pos"][k] in r["commit"]
                           for k, c in enumerate(r["conf"]))
        assert rem == 0 and sorted(seen) == list(range(1, cfg.B))
