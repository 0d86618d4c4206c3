"""Drafting and verify with the vocabulary split over GPUs (tensor-parallel serving).

"DFlash + Spec V2 深度解析", §3.3 serves the target with tensor parallelism
(--tp-size 8).  With the LM head split by vocabulary, the only exchange of
the draft hot path is one all-gather per denoising step (and one per verify)
of a fixed-size record per row and rank: each rank reduces its vocabulary
shard to (max, argmax id, sum of exp) per masked row (16 bytes), or to
(max, argmax id) per target-logit row (8 bytes), and every rank merges all
ranks' records, shards in vocabulary order, to the same tokens.  The
library's kernels do the reductions and the merge; this module only orders
the calls around the all-gather.

One process per GPU (torch.distributed, backend "nccl").  `gather` is the
exchange: by default an all-gather over the process group on the current
stream; tests pass their own to emulate ranks on one device.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

from . import dflash as D

Gather = Callable[[torch.Tensor], torch.Tensor]


def shard_bounds(V: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous vocabulary shards in rank order: sizes differ by at most one row."""
    if world < 1 or V < world:
        raise ValueError("need 1 <= world <= V")
    base, extra = divmod(V, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def all_gather(group=None) -> Gather:
    """The exchange over a torch.distributed process group: stacks every rank's
    tensor along a new leading dimension, in rank order."""
    import torch.distributed as dist

    def gather(local: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(out, local.contiguous(), group=group)
        else:  # gloo (host tests)
            dist.all_gather(list(out.unbind(0)), local.contiguous(), group=group)
        return out

    return gather


def draft_block(model: "D.Model", anchor: torch.Tensor, ctx_len: torch.Tensor,
                k_cache: torch.Tensor, v_cache: torch.Tensor, B: int, n_steps: int,
                draft_tokens: torch.Tensor, ws: torch.Tensor, gather: Gather,
                commit_step: Optional[torch.Tensor] = None, stream=None) -> None:
    """Greedy draft of a batch on a vocabulary-shard model: begin, then per step the
    shard forward, the exchange of the per-row records and the merged commit,
    then end.  Every rank calls it with the same inputs."""
    batch = anchor.numel()
    D.draft_begin(model, anchor, ctx_len, k_cache.shape[3], B, n_steps, ws, stream)
    for t in range(n_steps):
        rows = D.draft_rows(batch, B, n_steps, t)
        mine = torch.empty((rows, 4), dtype=torch.float32, device=k_cache.device)
        D.draft_forward_shard(model, ctx_len, k_cache, v_cache, B, n_steps, t, mine, ws, stream)
        D.draft_commit_shards(model, gather(mine), batch, B, n_steps, t, ws, stream)
    D.draft_end(model, B, n_steps, draft_tokens, ws, commit_step, stream)


def verify(logits_shard: torch.Tensor, vocab_offset: int, V: int, draft_tokens: torch.Tensor,
           out_tokens: torch.Tensor, out_len: torch.Tensor, seq_lens: torch.Tensor,
           accept_len: torch.Tensor, next_anchor: torch.Tensor, ws: torch.Tensor,
           gather: Gather, stream=None) -> None:
    """Greedy verify with this rank's target-logit columns [batch, B, Vs] (global
    ids vocab_offset ..): the per-row shard argmax, the exchange, the merged
    accept.  Every rank ends with the same outputs."""
    batch, B, _ = logits_shard.shape
    mine = torch.empty((batch * B, 2), dtype=torch.float32, device=logits_shard.device)
    D.verify_shard(logits_shard, vocab_offset, mine, ws, stream)
    D.verify_merge(gather(mine), draft_tokens, V, out_tokens, out_len, seq_lens, accept_len,
                   next_anchor, ws, stream)

