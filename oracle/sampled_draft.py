"""Plain fp64 restatement of block drafting under temperature sampling.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Slow and direct on
purpose: the draft forward is the greedy oracle's (``dflash_oracle``); only the
token choice and the confidence change.

Sources (page title, then section):

* "DFlash + Spec V2 深度解析", §2.3 块扩散: the block starts as [anchor, MASK,
  ..., MASK]; each forward predicts every masked position; 2-3 rounds fix the
  positions step by step, most confident first.
* "DFlash: Block Diffusion for Flash Speculative Decoding" (study notes),
  §消融实验结论: drafting holds up under high-temperature sampling.

The pages say nothing about how a diffusion draft samples.  The reading taken is
the sampled counterpart of the greedy rule:

* at step t every still-masked position j draws a candidate x_j from
  softmax(Y_j / tau) (Y_j = the LM-head logits at j in this step) by
  Gumbel-max: argmax_v (Y_jv / tau - log(-log U'_v)), ties to the lowest
  index, U' from Philox4x64-10 stream 2 under key (seed, 0).  The uniform for
  vocabulary entry v is draw n = (t * B + j) * V + v: word n % 4 of counter
  (offset, request, 2, n // 4), mapped as ((w >> 11) + 1/2) 2^-53;
* its confidence is the model's own (untempered) probability of the drawn
  token, softmax(Y_j)(x_j): temperature changes what is drawn, not how sure
  the model is of it, and as tau -> 0 the draw and its confidence become the
  greedy argmax and max-probability;
* the ceil(remaining / steps left) most confident positions commit their drawn
  tokens (ties to the lower position);
* the logits of the step that commits position j are the draft's
  distribution q_j for sampled verify.

With one step (s = 1), every position keeps its draw, so d_j is an exact draw
from q_j.  With s > 1, choosing positions by the drawn token's own
probability conditions the kept token on being confident.  q_j is then the
distribution it was drawn from, not the distribution given that it was kept.
"""

from __future__ import annotations

from typing import Optional

import numpy as np

from .dflash_oracle import Weights64, commit_count, draft_hidden, select_commits
from .sampled_verify import (gumbel_argmax, log_softmax, neg_log_uniform_open, philox_words,
                             uniform_open)

__all__ = ["STREAM_DRAFT", "draft_draw_uniforms", "draft_draw_exponentials", "sampled_draft_block"]

STREAM_DRAFT = 2


def draft_draw_uniforms(seed: int, offset: int, request: int, step: int, pos: int, B: int,
                        V: int) -> np.ndarray:
    """U'_v, v < V, of position `pos` at denoising step `step` (stream 2)."""
    n0 = (step * B + pos) * V
    return uniform_open(philox_words(seed, offset, request, STREAM_DRAFT, n0 + np.arange(V)))


def draft_draw_exponentials(seed: int, offset: int, request: int, step: int, pos: int, B: int,
                            V: int) -> np.ndarray:
    """-ln U'_v, v < V, of the same draws, exact (neg_log_uniform_open)."""
    n0 = (step * B + pos) * V
    return neg_log_uniform_open(philox_words(seed, offset, request, STREAM_DRAFT,
                                             n0 + np.arange(V)))


def sampled_draft_block(anchor: int, T: int, caches, W: Weights64, cfg, tau: float, seed: int,
                        offset: int, request: int, steps: Optional[int] = None):
    """Draft one block for one request under temperature tau.

    Returns (tokens [B], draft_logits [B, V] with row 0 zero, records), where
    draft_logits[j] holds the logits of the step that committed position j and
    records[t] = {"pos", "draw", "conf", "commit", "logits"} for step t.
    """
    steps = cfg.steps if steps is None else steps
    B, V = cfg.B, cfg.V
    tokens = np.full(B, cfg.mask_id, dtype=np.int64)
    tokens[0] = anchor
    masked = list(range(1, B))
    q_logits = np.zeros((B, V))
    records = []
    for t in range(steps):
        z = draft_hidden(tokens, T, caches, W, cfg)
        Y = W.lm_logits(z[masked])
        lp = log_softmax(Y, tau)
        lp1 = log_softmax(Y, 1.0)
        draws, confs = [], []
        for i, j in enumerate(masked):
            x, _ = gumbel_argmax(lp[i], draft_draw_exponentials(seed, offset, request, t, j, B, V))
            draws.append(x)
            confs.append(float(np.exp(lp1[i, x])))
        k = commit_count(len(masked), steps - t)
        commit = select_commits(masked, confs, k)
        idx = {p: i for i, p in enumerate(masked)}
        for p in commit:
            tokens[p] = draws[idx[p]]
            q_logits[p] = Y[idx[p]]
        records.append({"pos": list(masked), "draw": draws, "conf": confs, "commit": commit,
                        "logits": Y})
        masked = [p for p in masked if p not in commit]
    return tokens, q_logits, records
