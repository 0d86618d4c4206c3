"""Plain fp64 restatement of injection into, and drafting from, a paged K/V cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "DFlash: Block Diffusion for Flash Speculative Decoding" (study notes),
§2 KV 注入: context features are projected into the draft's K/V once, cached for
reuse, and support prefix sharing.  An injected K/V row depends only on the
target hidden state at its position and on the position.  Requests whose
contexts share a prefix therefore produce the same rows for it, and can share
the pages that hold them.

Layout (the reading taken; the pages give none):

* Each layer has a pool of pages, K_pool and V_pool of shape
  [L, n_pages, nkv, P, hd], with P positions per page.
* Request r maps context position p to page table[r, p // P], slot p % P.
* A table entry of -1 is unmapped; so is any id outside [0, n_pages).
* Injection of a request touching an unmapped page writes nothing for that
  request and reports STATUS_PAGE.
* The draft reads positions 0..T_r-1 through the table; a request whose table
  does not map all of them is reported the same way.

The arithmetic is the contiguous oracle's (``dflash_oracle``): gathering the
pages of a request gives exactly its contiguous cache.
"""

from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np

from .dflash_oracle import Weights64, draft_block, inject_kv_requests

__all__ = ["STATUS_OK", "STATUS_PAGE", "page_of", "gather_caches", "inject_kv_paged",
           "draft_block_paged"]

STATUS_OK = 0
STATUS_PAGE = 4


def page_of(table_r, p: int, P: int, n_pages: int) -> int:
    """Page id holding position p of a request, or -1 when unmapped."""
    k = p // P
    if k >= len(table_r):
        return -1
    pg = int(table_r[k])
    return pg if 0 <= pg < n_pages else -1


def gather_caches(K_pool: np.ndarray, V_pool: np.ndarray, table_r, T: int, P: int):
    """Contiguous per-layer caches [(K [T, nkv, hd], V [T, nkv, hd]), ...] of one
    request, or None when a position below T is unmapped."""
    L, n_pages = K_pool.shape[0], K_pool.shape[1]
    pages = [page_of(table_r, p, P, n_pages) for p in range(T)]
    if any(pg < 0 for pg in pages):
        return None
    slots = [p % P for p in range(T)]
    out = []
    for l in range(L):
        K = np.stack([K_pool[l, pages[p], :, slots[p], :] for p in range(T)]) if T else \
            np.zeros((0, K_pool.shape[2], K_pool.shape[4]))
        V = np.stack([V_pool[l, pages[p], :, slots[p], :] for p in range(T)]) if T else \
            np.zeros((0, V_pool.shape[2], V_pool.shape[4]))
        out.append((K, V))
    return out


def inject_kv_paged(taps, cu_rows, start_pos, table, P: int, W: Weights64, cfg,
                    K_pool: np.ndarray, V_pool: np.ndarray):
    """Inject a packed batch into the page pools (copies are returned).

    Rows of request r go to positions start_pos[r] + 0, 1, ... through table[r].
    Returns (K_pool, V_pool, status [batch]).
    """
    K_pool = np.array(K_pool, dtype=np.float64, copy=True)
    V_pool = np.array(V_pool, dtype=np.float64, copy=True)
    n_pages = K_pool.shape[1]
    rows = inject_kv_requests(taps, cu_rows, start_pos, W, cfg)
    b = len(start_pos)
    status = np.zeros(b, dtype=np.int64)
    for r in range(b):
        pos = rows[(0, r)][0]
        pages = [page_of(table[r], int(p), P, n_pages) for p in pos]
        if any(pg < 0 for pg in pages):
            status[r] = STATUS_PAGE
            continue
        for l in range(cfg.L):
            _, K, V = rows[(l, r)]
            for i, p in enumerate(pos):
                K_pool[l, pages[i], :, int(p) % P, :] = K[i]
                V_pool[l, pages[i], :, int(p) % P, :] = V[i]
    return K_pool, V_pool, status


def draft_block_paged(anchor: int, T: int, K_pool, V_pool, table_r, P: int, W: Weights64, cfg,
                      steps=None):
    """Greedy draft of one request reading its context through the page table;
    (None, None) when the table leaves a position below T unmapped."""
    caches = gather_caches(K_pool, V_pool, table_r, T, P)
    if caches is None:
        return None, None
    return draft_block(anchor, T, caches, W, cfg, steps=steps)
