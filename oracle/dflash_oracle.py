"""Plain fp64 restatement of DFlash block-diffusion drafting and greedy verify.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Slow and direct on
purpose: every function computes its definition in float64 with NumPy, with a
library matmul as the only building block, no blocking, fusion or reordering.
Inputs in bf16 or fp32 convert exactly to float64; nothing is rounded in
between.

Sources (page title, then section):

* "DFlash: Block Diffusion for Flash Speculative Decoding" (study notes on
  arXiv 2602.06036): §整体架构 (target -> multi-layer hidden states -> context
  features -> KV injection -> block diffusion draft -> verify), §1 上下文特征提取,
  §2 KV 注入, §3 块级扩散解码, §Immediate Materialization (layer-batched linear
  projections).
* "DFlash + Spec V2 深度解析": §2.2 KV 注入 (inject into every draft layer's KV
  cache), §2.3 块扩散 (all-[MASK] block, one forward predicts every position,
  2-3 denoising rounds), §4.2 (block 8, two diffusion steps).
* "DFlash：用“块扩散”魔法" (blog): §核心创新 inference sketch
  (generate_block(context, block_size) then verify(context, draft_block)) and
  §2 Flash Verification (decide_acceptance(logits, draft_block)).

The pages give no formulas.  Where they leave a step open this file takes the
plain reading listed in the design notes: concat of taps in ascending order ->
fc (no bias) -> RMSNorm (eps 1e-6) as the context feature; each draft layer's
own Wk/Wv project the features into its cache, K rotated by rotate-half RoPE
(base 1e6) at the absolute position; pre-norm attention + SwiGLU layers; GQA
with query head i reading kv head i // (nq/nkv); no mask inside the block;
argmax ties to the lowest vocabulary index; confidence = softmax max-probability;
greedy verify by longest matching prefix.
"""

from __future__ import annotations

import itertools
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "as_f64",
    "Weights64",
    "rms_norm",
    "rope_cos_sin",
    "apply_rope",
    "silu",
    "context_features",
    "inject_kv",
    "inject_kv_requests",
    "block_attention",
    "draft_layer",
    "draft_hidden",
    "lm_head_stats",
    "commit_count",
    "select_commits",
    "valid_commit_sets",
    "draft_step",
    "draft_block",
    "row_argmax",
    "accept_length",
    "verify_request",
    "verify_batch",
    "VERIFY_OK",
    "VERIFY_OUT_CAP",
    "VERIFY_TOKEN_RANGE",
]


# --------------------------------------------------------------------------
# conversions
# --------------------------------------------------------------------------

def as_f64(a) -> np.ndarray:
    """Exact conversion of a torch tensor (any float type) or array to float64."""
    if hasattr(a, "detach"):
        import torch  # only for the conversion

        a = a.detach().to("cpu")
        if a.dtype in (torch.bfloat16, torch.float16):
            a = a.to(torch.float32)
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def _as_int(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.asarray(a, dtype=np.int64)


class Weights64:
    """Lazy float64 view of the draft weights dict (see ``synth.make_weights``).

    Matrices are kept in [out_features, in_features] layout, so a linear map is
    ``x @ W.T``.  Converted matrices are memoised; the embedding table and the
    LM head are read in slices instead, to bound memory.
    """

    def __init__(self, w: Dict, cfg):
        self.w = w
        self.cfg = cfg
        self._cache = {}

    def mat(self, *key) -> np.ndarray:
        if key not in self._cache:
            obj = self.w
            for k in key:
                obj = obj[k]
            self._cache[key] = as_f64(obj)
        return self._cache[key]

    def layer(self, l: int, name: str) -> np.ndarray:
        return self.mat("layers", l, name)

    def emb_rows(self, tokens: np.ndarray) -> np.ndarray:
        import torch

        idx = torch.as_tensor(np.asarray(tokens, dtype=np.int64))
        return as_f64(self.w["emb"].index_select(0, idx))

    def lm_logits(self, z: np.ndarray, chunk: int = 16384) -> np.ndarray:
        """z @ W_lm.T, reading W_lm in row slices."""
        W = self.w["W_lm"]
        V = W.shape[0]
        out = np.empty((z.shape[0], V), dtype=np.float64)
        for s in range(0, V, chunk):
            e = min(V, s + chunk)
            out[:, s:e] = z @ as_f64(W[s:e]).T
        return out


# --------------------------------------------------------------------------
# elementwise pieces (readings: the pages name no normalisation or position code)
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def rope_cos_sin(pos, hd: int, base: float):
    """cos/sin of angle p * base^(-2i/hd), i = 0..hd/2-1, for each position p."""
    pos = np.asarray(pos, dtype=np.float64).reshape(-1)
    i = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)
    ang = pos[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE: pair (i, i+hd/2) is turned by angle p*theta_i.

    x has shape [n, heads, hd]; pos has n entries.
    """
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    h = hd // 2
    c, s = rope_cos_sin(pos, hd, base)
    c = c[:, None, :]
    s = s[:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


# --------------------------------------------------------------------------
# context feature extraction and KV injection
# --------------------------------------------------------------------------

def context_features(taps: Sequence, W_fc, g_ctx, eps: float) -> np.ndarray:
    """Fuse the tapped target hidden states of each row into one feature vector.

    "DFlash: Block Diffusion for Flash Speculative Decoding", §1 上下文特征提取:
    multi-layer target hidden states are fused into a compact context feature.
    Reading: concatenate along features in ascending tap order, apply the fc
    map (no bias), then RMSNorm with gain g_ctx.  Returns c [n, d].
    """
    X = np.concatenate([as_f64(t) for t in taps], axis=1)
    u = X @ as_f64(W_fc).T
    return rms_norm(u, as_f64(g_ctx), eps)


def inject_kv(c: np.ndarray, pos, Wk, Wv, nkv: int, hd: int, base: float):
    """Project context features into one draft layer's K/V cache entries.

    "DFlash: Block Diffusion for Flash Speculative Decoding", §2 KV 注入, and
    "DFlash + Spec V2 深度解析", §2.2: the features are written into every draft
    layer's K/V (the draft attends to them instead of re-encoding the context).
    K_l[p] = RoPE(c[p] Wk_l^T, p), V_l[p] = c[p] Wv_l^T.  Returns K, V as
    [n, nkv, hd].
    """
    n = c.shape[0]
    K = (c @ as_f64(Wk).T).reshape(n, nkv, hd)
    V = (c @ as_f64(Wv).T).reshape(n, nkv, hd)
    return apply_rope(K, pos, base), V


def inject_kv_requests(taps, cu_rows, start_pos, W: Weights64, cfg):
    """Injection for a packed batch of requests.

    Rows cu_rows[r]..cu_rows[r+1]-1 belong to request r and sit at positions
    start_pos[r] + 0, 1, ...  Every draft layer is projected from the same
    features ("Immediate Materialization": layer-batched projections).
    Returns {(l, r): (positions, K [n_r, nkv, hd], V [n_r, nkv, hd])}.
    """
    cu = _as_int(cu_rows)
    st = _as_int(start_pos)
    c = context_features(taps, W.mat("W_fc"), W.mat("g_ctx"), cfg.eps)
    out = {}
    for r in range(len(st)):
        rows = np.arange(cu[r], cu[r + 1])
        pos = st[r] + (rows - cu[r])
        for l in range(cfg.L):
            K, V = inject_kv(c[rows], pos, W.layer(l, "Wk"), W.layer(l, "Wv"), cfg.nkv, cfg.hd,
                             cfg.rope_base)
            out[(l, r)] = (pos, K, V)
    return out


# --------------------------------------------------------------------------
# block diffusion draft forward
# --------------------------------------------------------------------------

def block_attention(q: np.ndarray, K_ctx: np.ndarray, V_ctx: np.ndarray, k_blk: np.ndarray,
                    v_blk: np.ndarray) -> np.ndarray:
    """Attention of the block queries over context keys followed by the block's own keys.

    "DFlash + Spec V2 深度解析", §2.3: the whole block is predicted in one
    forward, so no mask is applied inside the block (every block position sees
    every other) and every block position sees the whole injected context.
    q [B, nq, hd]; K_ctx/V_ctx [T, nkv, hd]; k_blk/v_blk [B, nkv, hd].
    Query head i reads kv head i // (nq/nkv).  Returns o [B, nq, hd].
    """
    B, nq, hd = q.shape
    nkv = k_blk.shape[1]
    group = nq // nkv
    K = np.concatenate([K_ctx, k_blk], axis=0)
    V = np.concatenate([V_ctx, v_blk], axis=0)
    o = np.empty_like(q)
    for i in range(nq):
        j = i // group
        S = q[:, i, :] @ K[:, j, :].T / math.sqrt(hd)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        o[:, i, :] = P @ V[:, j, :]
    return o


def draft_layer(x: np.ndarray, pos, K_ctx, V_ctx, W: Weights64, l: int, cfg) -> np.ndarray:
    """One pre-norm draft layer over the block rows of one request.

    h = RMSNorm(x; g_in); q, k, v = h Wq^T, h Wk^T, h Wv^T with RoPE on q and k;
    x += attention(...) Wo^T; h2 = RMSNorm(x; g_post); x += (silu(h2 Wg^T) * (h2 Wu^T)) Wd^T.
    """
    B = x.shape[0]
    h = rms_norm(x, W.layer(l, "g_in"), cfg.eps)
    q = apply_rope((h @ W.layer(l, "Wq").T).reshape(B, cfg.nq, cfg.hd), pos, cfg.rope_base)
    k = apply_rope((h @ W.layer(l, "Wk").T).reshape(B, cfg.nkv, cfg.hd), pos, cfg.rope_base)
    v = (h @ W.layer(l, "Wv").T).reshape(B, cfg.nkv, cfg.hd)
    o = block_attention(q, K_ctx, V_ctx, k, v)
    x = x + o.reshape(B, cfg.nq * cfg.hd) @ W.layer(l, "Wo").T
    h2 = rms_norm(x, W.layer(l, "g_post"), cfg.eps)
    act = silu(h2 @ W.layer(l, "Wg").T) * (h2 @ W.layer(l, "Wu").T)
    return x + act @ W.layer(l, "Wd").T


def draft_hidden(tokens, T: int, caches, W: Weights64, cfg) -> np.ndarray:
    """Final-normed hidden states z [B, d] of one request's block.

    tokens: the B block tokens (anchor, then committed tokens or [MASK]) at
    positions T..T+B-1.  caches[l] = (K_ctx [T, nkv, hd], V_ctx [T, nkv, hd]).
    """
    tokens = _as_int(tokens)
    B = tokens.shape[0]
    pos = T + np.arange(B)
    x = W.emb_rows(tokens)
    for l in range(cfg.L):
        Kc, Vc = caches[l]
        x = draft_layer(x, pos, Kc, Vc, W, l, cfg)
    return rms_norm(x, W.mat("g_final"), cfg.eps)


def lm_head_stats(z: np.ndarray, W: Weights64, band: float = 0.05, keep_logits: bool = False):
    """Greedy prediction per row: argmax token, softmax max-probability, top-2 margin.

    tok = argmax_v logits (lowest v on ties); conf = 1 / sum_v exp(logit_v - max);
    margin = top-1 logit minus top-2 logit; cand = every token within ``band``
    of the maximum (the tokens a near-tie admits).
    """
    logits = W.lm_logits(z)
    tok = np.argmax(logits, axis=1)
    mx = logits[np.arange(len(tok)), tok]
    conf = 1.0 / np.exp(logits - mx[:, None]).sum(axis=1)
    top2 = np.partition(logits, -2, axis=1)[:, -2:]
    margin = top2[:, 1] - top2[:, 0]
    cand = [np.nonzero(logits[i] >= mx[i] - band)[0] for i in range(len(tok))]
    out = {"tok": tok, "conf": conf, "margin": margin, "max": mx, "cand": cand}
    if keep_logits:
        out["logits"] = logits
    return out


def commit_count(n_masked: int, steps_left: int) -> int:
    """Positions committed at a denoising step: ceil(remaining / steps left).

    "DFlash + Spec V2 深度解析", §2.3: 2-3 rounds fix the positions step by step;
    the per-step count spreads the masked positions evenly over the steps left.
    """
    return -(-n_masked // steps_left)


def select_commits(pos: Sequence[int], conf: Sequence[float], k: int) -> List[int]:
    """The k most confident masked positions, ties to the lower position."""
    order = sorted(range(len(pos)), key=lambda i: (-conf[i], pos[i]))
    return sorted(pos[i] for i in order[:k])


def valid_commit_sets(pos: Sequence[int], conf: Sequence[float], k: int, rel_band: float):
    """Every size-k commit set that differs from the exact choice only inside the band.

    A set S is admitted when no excluded position is more confident than an
    included one by more than ``rel_band`` relative: min_{S} conf >=
    (1 - rel_band) * max_{not S} conf.
    """
    n = len(pos)
    if k >= n:
        return [sorted(pos)]
    sets = []
    for S in itertools.combinations(range(n), k):
        inn = min(conf[i] for i in S)
        out = max(conf[i] for i in range(n) if i not in S)
        if inn >= (1.0 - rel_band) * out:
            sets.append(sorted(pos[i] for i in S))
    return sets


def draft_step(tokens_batch, masked_batch, T_list, caches_batch, W: Weights64, cfg,
               keep_logits: bool = False):
    """One denoising forward for several requests: stats at every still-masked position.

    tokens_batch[r]: current B tokens; masked_batch[r]: list of masked positions.
    Returns a list (per request) of dicts from ``lm_head_stats`` plus 'pos'.
    """
    out = []
    for r, toks in enumerate(tokens_batch):
        z = draft_hidden(toks, T_list[r], caches_batch[r], W, cfg)
        m = list(masked_batch[r])
        st = lm_head_stats(z[m], W, keep_logits=keep_logits) if m else None
        if st is not None:
            st["pos"] = m
        out.append(st)
    return out


def draft_block(anchor: int, T: int, caches, W: Weights64, cfg, steps: Optional[int] = None,
                keep: bool = False):
    """Draft one block for one request (greedy, no branching).

    "DFlash + Spec V2 深度解析", §2.3: start from [anchor, MASK, ..., MASK]; each
    forward predicts every masked position; step t commits the
    ceil(remaining / (s - t)) most confident positions to their argmax token.
    With s = 1 every masked position takes its argmax at once.
    Returns (tokens [B], records) where records[t] holds the step's stats and
    commit list.
    """
    steps = cfg.steps if steps is None else steps
    B = cfg.B
    tokens = np.full(B, cfg.mask_id, dtype=np.int64)
    tokens[0] = anchor
    masked = list(range(1, B))
    records = []
    for t in range(steps):
        st = draft_step([tokens], [masked], [T], [caches], W, cfg, keep_logits=keep)[0]
        k = commit_count(len(masked), steps - t)
        commit = select_commits(st["pos"], st["conf"], k)
        idx = {p: i for i, p in enumerate(st["pos"])}
        for p in commit:
            tokens[p] = st["tok"][idx[p]]
        records.append({"stats": st, "commit": commit})
        masked = [p for p in masked if p not in commit]
    return tokens, records


# --------------------------------------------------------------------------
# greedy verify
# --------------------------------------------------------------------------

VERIFY_OK = 0
VERIFY_OUT_CAP = 1
VERIFY_TOKEN_RANGE = 2


def row_argmax(logits) -> np.ndarray:
    """argmax over the last axis; ties go to the lowest index (first maximum)."""
    return np.argmax(as_f64(logits), axis=-1)


def accept_length(g: Sequence[int], draft: Sequence[int]) -> int:
    """Longest prefix with g[i] == draft[i+1]; at most B-1.

    "DFlash：用“块扩散”魔法", §2 Flash Verification: the target scores context +
    block in one pass and decide_acceptance keeps the draft tokens it agrees
    with; greedy reading: row i of the target logits predicts the token after
    block position i.
    """
    B = len(draft)
    a = 0
    while a < B - 1 and int(g[a]) == int(draft[a + 1]):
        a += 1
    return a


def verify_request(logits, draft):
    """(a, emitted tokens d_1..d_a followed by the bonus g_a, bonus) for one request."""
    g = row_argmax(logits)
    d = _as_int(draft)
    a = accept_length(g, d)
    emitted = [int(t) for t in d[1:a + 1]] + [int(g[a])]
    return a, emitted, int(g[a]), g


def verify_batch(logits, draft, out_tokens, out_len, out_cap: int, seq_lens):
    """Greedy verify for a batch, with compaction into per-request output buffers.

    For request r: a = accept length, emit d_1..d_a and the bonus g_a at
    out_tokens[r, out_len[r] : out_len[r]+a+1], then out_len += a+1,
    seq_lens += a+1, next_anchor = g_a.  A request whose draft holds a token
    outside [0, V) or whose output would pass out_cap writes nothing and
    reports a status (VERIFY_TOKEN_RANGE, VERIFY_OUT_CAP).
    Returns dict with updated copies and per-request accept/next_anchor/status.
    """
    L = as_f64(logits)
    d = _as_int(draft)
    b, B, V = L.shape
    out_tokens = _as_int(out_tokens).copy()
    out_len = _as_int(out_len).copy()
    seq = _as_int(seq_lens).copy()
    accept = np.full(b, -1, dtype=np.int64)
    nxt = np.full(b, -1, dtype=np.int64)
    status = np.zeros(b, dtype=np.int64)
    argmax = np.argmax(L, axis=-1)
    for r in range(b):
        if np.any(d[r] < 0) or np.any(d[r] >= V):
            status[r] = VERIFY_TOKEN_RANGE
            continue
        a, emitted, bonus, _ = verify_request(L[r], d[r])
        if out_len[r] + a + 1 > out_cap:
            status[r] = VERIFY_OUT_CAP
            continue
        out_tokens[r, out_len[r]:out_len[r] + a + 1] = emitted
        out_len[r] += a + 1
        seq[r] += a + 1
        accept[r] = a
        nxt[r] = bonus
    return {"out_tokens": out_tokens, "out_len": out_len, "seq_lens": seq, "accept": accept,
            "next_anchor": nxt, "status": status, "argmax": argmax}
