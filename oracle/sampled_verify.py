"""Plain fp64 restatement of sampled (temperature) verify of a drafted block.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Slow and direct on
purpose; float64 NumPy throughout, no blocking, fusion or reordering.

Sources (page title, then section):

* "DFlash: Block Diffusion for Flash Speculative Decoding" (study notes on
  arXiv 2602.06036): §消融实验结论 (drafting stays efficient under
  high-temperature sampling) and §与 Speculative Decoding 系列的关系 (DFlash
  descends from speculative decoding, Leviathan et al., 2023).
* "DFlash：用“块扩散”魔法" (blog), §2 Flash Verification: classic verification
  compares the target's conditional probabilities with the draft model's, and
  decide_acceptance(logits, draft_block) keeps a prefix of the block.

The pages state no acceptance rule for sampling.  The reading taken is standard
speculative sampling: with p_i = softmax(Z_i / tau), the target's distribution
for the token after block position i, and q_j = softmax(Y_j / tau), the draft's
distribution for block position j:

* for i = 0, 1, ..., B-2 in order, draft token x = d_{i+1} is accepted when
  U_i < p_i(x) / q_{i+1}(x) (U_i uniform in [0, 1)); the comparison is taken
  in the log domain (log U_i < log p_i(x) - log q_{i+1}(x)), so a vanishing
  q_{i+1}(x) accepts instead of dividing by zero;
* at the first rejection, a = i and the last token is drawn from
  max(0, p_i - q_{i+1}) (renormalised); with no rejection, a = B-1 and the last
  token is drawn from p_{B-1};
* emit d_1..d_a then the drawn token; out_len and seq_lens grow by a+1; the
  drawn token is the next anchor.

Draws: the token is the Gumbel-max argmax_v (log w_v + G_v) over the (possibly
unnormalised) weights w_v > 0, G_v = -log(-log U'_v), ties to the lowest index.
Every uniform comes from Philox4x64-10 (Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC 2011) under key (seed, 0).
Counter words are (offset, request, stream, n). The output word n % 4 of
counter n // 4 gives U_i (stream 0, n = i) or U'_v (stream 1, n = v).
A 64-bit word w maps to U = (w >> 11) * 2^-53 in [0, 1) and
U' = ((w >> 11) + 1/2) * 2^-53 in (0, 1).
"""

from __future__ import annotations

from typing import Dict, Sequence

import numpy as np

__all__ = [
    "PHILOX_M",
    "PHILOX_W",
    "philox4x64",
    "philox_words",
    "uniform_closed_open",
    "uniform_open",
    "STREAM_ACCEPT",
    "STREAM_DRAW",
    "accept_uniforms",
    "draw_uniforms",
    "draw_exponentials",
    "neg_log_uniform_open",
    "log_softmax",
    "gumbel_argmax",
    "residual_log_weights",
    "sampled_verify_request",
    "sampled_verify_batch",
]

# Philox4x64 round multipliers and Weyl key increments (golden ratio and sqrt(3) - 1)
PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)
_MASK64 = (1 << 64) - 1
_MASK32 = np.uint64(0xFFFFFFFF)

STREAM_ACCEPT = 0
STREAM_DRAW = 1


def _mulhilo(a: np.ndarray, m: int):
    """(high, low) 64-bit words of the 128-bit products a * m, element-wise."""
    a = a.astype(np.uint64)
    a_lo, a_hi = a & _MASK32, a >> np.uint64(32)
    m_lo, m_hi = np.uint64(m & 0xFFFFFFFF), np.uint64(m >> 32)
    with np.errstate(over="ignore"):
        ll = a_lo * m_lo
        lh = a_lo * m_hi
        hl = a_hi * m_lo
        hh = a_hi * m_hi
        mid = (ll >> np.uint64(32)) + (lh & _MASK32) + (hl & _MASK32)
        hi = hh + (lh >> np.uint64(32)) + (hl >> np.uint64(32)) + (mid >> np.uint64(32))
        lo = a * np.uint64(m)
    return hi, lo


def philox4x64(counter, key, rounds: int = 10) -> np.ndarray:
    """Philox4x64 block function on counters of shape [..., 4] (uint64) and a key of two
    64-bit words; returns [..., 4] uint64.

    One round maps (c0, c1, c2, c3) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
    hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the key grows by the Weyl increments
    between rounds.
    """
    c = np.array(counter, dtype=np.uint64).copy()
    k0, k1 = int(key[0]) & _MASK64, int(key[1]) & _MASK64
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + PHILOX_W[0]) & _MASK64
            k1 = (k1 + PHILOX_W[1]) & _MASK64
        hi0, lo0 = _mulhilo(c[..., 0], PHILOX_M[0])
        hi1, lo1 = _mulhilo(c[..., 2], PHILOX_M[1])
        n0 = hi1 ^ c[..., 1] ^ np.uint64(k0)
        n2 = hi0 ^ c[..., 3] ^ np.uint64(k1)
        c = np.stack([n0, lo1, n2, lo0], axis=-1)
    return c


def philox_words(seed: int, offset: int, request: int, stream: int, n) -> np.ndarray:
    """64-bit word n (array) of the stream: word n % 4 of counter
    (offset, request, stream, n // 4) under key (seed, 0)."""
    n = np.asarray(n, dtype=np.uint64)
    ctr = np.stack([np.full(n.shape, offset, dtype=np.uint64),
                    np.full(n.shape, request, dtype=np.uint64),
                    np.full(n.shape, stream, dtype=np.uint64),
                    n >> np.uint64(2)], axis=-1)
    out = philox4x64(ctr, (seed, 0))
    return np.take_along_axis(out, (n & np.uint64(3)).astype(np.int64)[..., None], axis=-1)[..., 0]


def uniform_closed_open(w) -> np.ndarray:
    """U = (w >> 11) * 2^-53: the top 53 bits as a double in [0, 1)."""
    return (np.asarray(w, dtype=np.uint64) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def uniform_open(w) -> np.ndarray:
    """U' = ((w >> 11) + 1/2) * 2^-53: a double in (0, 1), never 0 or 1."""
    return ((np.asarray(w, dtype=np.uint64) >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def neg_log_uniform_open(w) -> np.ndarray:
    """E = -ln U' for U' = ((w >> 11) + 1/2) * 2^-53, the exponential variate of a
    Gumbel draw, without rounding U' first.  Below 1/2, U' = (k + 1/2) 2^-53 is
    exact in float64 and E = -log U'.  From 1/2 up, U' needs 54 bits, but
    1 - U' = (2^53 - 1 - k + 1/2) 2^-53 is exact and E = -log1p(-(1 - U')).
    (Rounding U' to float64 would drop its last bit there and turn the top word
    into U' = 1, E = 0.)"""
    k = np.asarray(w, dtype=np.uint64) >> np.uint64(11)
    lo = k < np.uint64(1 << 52)
    u = (k.astype(np.float64) + 0.5) * 2.0 ** -53
    m = ((np.uint64((1 << 53) - 1) - k).astype(np.float64) + 0.5) * 2.0 ** -53
    with np.errstate(divide="ignore"):
        return np.where(lo, -np.log(u), -np.log1p(-m))


def accept_uniforms(seed: int, offset: int, request: int, n: int) -> np.ndarray:
    """U_0 .. U_{n-1} of a request (stream 0)."""
    return uniform_closed_open(philox_words(seed, offset, request, STREAM_ACCEPT, np.arange(n)))


def draw_uniforms(seed: int, offset: int, request: int, V: int) -> np.ndarray:
    """U'_0 .. U'_{V-1} of a request (stream 1), one per vocabulary entry."""
    return uniform_open(philox_words(seed, offset, request, STREAM_DRAW, np.arange(V)))


def draw_exponentials(seed: int, offset: int, request: int, V: int) -> np.ndarray:
    """-ln U'_0 .. -ln U'_{V-1} of a request (stream 1), exact (neg_log_uniform_open)."""
    return neg_log_uniform_open(philox_words(seed, offset, request, STREAM_DRAW, np.arange(V)))


def log_softmax(z, tau: float) -> np.ndarray:
    """log softmax(z / tau) over the last axis, in float64."""
    s = np.asarray(z, dtype=np.float64) / float(tau)
    m = np.max(s, axis=-1, keepdims=True)
    return s - m - np.log(np.sum(np.exp(s - m), axis=-1, keepdims=True))


def gumbel_argmax(logw: np.ndarray, e: np.ndarray):
    """Gumbel-max draw: argmax_v (logw_v - log E_v), E_v = -ln U'_v (so -log E_v is
    the Gumbel variate), over entries with a finite log-weight, ties to the lowest
    index.  Returns (index, the score array)."""
    score = np.where(np.isfinite(logw), logw - np.log(e), -np.inf)
    return int(np.argmax(score)), score


def residual_log_weights(lp: np.ndarray, lq: np.ndarray) -> np.ndarray:
    """log max(0, p - q) from log p and log q (-inf where p <= q):
    log p + log1p(-exp(log q - log p))."""
    out = np.full(lp.shape, -np.inf)
    pos = lp > lq
    out[pos] = lp[pos] + np.log1p(-np.exp(lq[pos] - lp[pos]))
    return out


def sampled_verify_request(Z, Y, draft, tau: float, seed: int, offset: int, request: int):
    """Sampled verify of one request.

    Z: target logits [B, V] (row i scores the token after block position i).
    Y: draft logits [B, V] (row j is the draft's distribution at block
    position j; row 0 is not used).  draft: [B] tokens, draft[0] the anchor.
    Returns a dict: a, emitted (d_1..d_a then the drawn token), token, and the
    quantities the decisions were taken on (log_rho, log_u, the draw's scores).
    """
    Z = np.asarray(Z, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    d = [int(t) for t in draft]
    B, V = Z.shape
    lp = log_softmax(Z, tau)
    lq = log_softmax(Y, tau)
    U = accept_uniforms(seed, offset, request, max(B - 1, 1))
    log_rho, log_u = [], []
    a = B - 1
    for i in range(B - 1):
        x = d[i + 1]
        lr = lp[i, x] - lq[i + 1, x]
        lu = np.log(U[i]) if U[i] > 0 else -np.inf
        log_rho.append(float(lr))
        log_u.append(float(lu))
        if not lu < lr:
            a = i
            break
    logw = residual_log_weights(lp[a], lq[a + 1]) if a < B - 1 else lp[B - 1]
    if not np.any(np.isfinite(logw)):
        logw = lp[a]  # p == q to the last bit: the residual is empty, draw from p
    tok, score = gumbel_argmax(logw, draw_exponentials(seed, offset, request, V))
    return {"a": a, "emitted": d[1:a + 1] + [tok], "token": tok, "log_rho": log_rho,
            "log_u": log_u, "score": score, "logw": logw}


VERIFY_OK = 0
VERIFY_OUT_CAP = 1
VERIFY_TOKEN_RANGE = 2


def sampled_verify_batch(Z, Y, draft, tau: float, seed: int, offset: int, out_tokens,
                         out_len, out_cap: int, seq_lens) -> Dict[str, np.ndarray]:
    """Sampled verify for a batch with compaction into per-request output buffers.

    Request r uses counter word 1 = r.  Outputs as in greedy verify: emitted
    tokens at out_tokens[r, out_len[r] : out_len[r]+a+1], out_len and seq_lens
    grow by a+1, accept = a, next_anchor = the drawn token.  A request whose
    draft holds a token outside [0, V) or whose output would pass out_cap writes
    nothing and reports VERIFY_TOKEN_RANGE / VERIFY_OUT_CAP.
    """
    Z = np.asarray(Z, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    d = np.asarray(draft, dtype=np.int64)
    b, B, V = Z.shape
    out_tokens = np.array(out_tokens, dtype=np.int64, copy=True)
    out_len = np.array(out_len, dtype=np.int64, copy=True)
    seq = np.array(seq_lens, dtype=np.int64, copy=True)
    accept = np.full(b, -1, dtype=np.int64)
    nxt = np.full(b, -1, dtype=np.int64)
    status = np.zeros(b, dtype=np.int64)
    detail = []
    for r in range(b):
        if np.any(d[r] < 0) or np.any(d[r] >= V):
            status[r] = VERIFY_TOKEN_RANGE
            detail.append(None)
            continue
        res = sampled_verify_request(Z[r], Y[r], d[r], tau, seed, offset, r)
        detail.append(res)
        a = res["a"]
        if out_len[r] + a + 1 > out_cap:
            status[r] = VERIFY_OUT_CAP
            continue
        out_tokens[r, out_len[r]:out_len[r] + a + 1] = res["emitted"]
        out_len[r] += a + 1
        seq[r] += a + 1
        accept[r] = a
        nxt[r] = res["token"]
    return {"out_tokens": out_tokens, "out_len": out_len, "seq_lens": seq, "accept": accept,
            "next_anchor": nxt, "status": status, "detail": detail}
