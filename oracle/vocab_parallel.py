"""Plain fp64 restatement of the LM-head statistics and verify argmax over a
vocabulary split into shards.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "DFlash + Spec V2 深度解析", §3.3 (the target is served with tensor
parallelism, --tp-size 8).  The pages give no split of the draft's LM head;
the reading taken is the plain one: rank k holds the contiguous vocabulary
shard [lo_k, hi_k), shards in rank order covering [0, V).  Per row a shard is
reduced to (largest logit, its lowest global id, sum over the shard of
exp(logit - largest)); the records of all shards, merged in shard order, give
the whole row's argmax (lowest id on ties) and softmax max-probability.  The
verify record is (largest logit, lowest global id).
"""

from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

__all__ = ["shard_record", "merge_records", "verify_shard_record", "merge_argmax"]


def shard_record(logits_row, lo: int, hi: int) -> Tuple[float, int, float]:
    """(max, lowest global id of the max, sum of exp(logit - max)) over columns [lo, hi)."""
    x = np.asarray(logits_row, dtype=np.float64)[lo:hi]
    j = int(np.argmax(x))
    m = float(x[j])
    return m, lo + j, float(np.exp(x - m).sum())


def merge_records(records: Sequence[Tuple[float, int, float]]) -> Tuple[int, float]:
    """Token and max-probability of a row from its shards' records, shards in order:
    the largest max wins (the lower id on equal maxima), and every shard's sum is
    rescaled to it."""
    M = max(r[0] for r in records)
    tok = min(r[1] for r in records if r[0] == M)
    total = sum(r[2] * np.exp(r[0] - M) for r in records)
    return tok, float(1.0 / total)


def verify_shard_record(logits_row, lo: int, hi: int) -> Tuple[float, int]:
    x = np.asarray(logits_row, dtype=np.float64)[lo:hi]
    j = int(np.argmax(x))
    return float(x[j]), lo + j


def merge_argmax(records: Sequence[Tuple[float, int]]) -> int:
    M = max(r[0] for r in records)
    return min(r[1] for r in records if r[0] == M)
