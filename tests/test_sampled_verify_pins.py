"""Pins for the sampled-verify oracle (oracle/sampled_verify.py).

Each check rests on something other than the oracle's own formulas:

* its Philox4x64-10 against NumPy's independent implementation
  (``numpy.random.Philox``);
* exact end points of the word-to-uniform maps;
* the speculative-sampling theorem: whatever the draft distribution, the
  first emitted token is distributed as the target's p_0.  This is a
  chi-square test over many requests, run through the oracle's own draws, and
  a planted mistake (drawing from p instead of the residual) must fail it;
* the closed-form acceptance rate 1 - TV(p, q);
* the tau -> 0 limit, which must reproduce greedy verify (itself pinned in
  test_oracle_pins.py);
* the sure-accept and sure-reject cases, and the output bookkeeping.
"""

from decimal import Decimal, localcontext

import numpy as np
import pytest
import scipy.stats

import oracle as O
import synth

SV = O.sampled_verify
M64 = (1 << 64) - 1


def _numpy_philox_block(key, ctr):
    """Philox4x64-10 output block for counter `ctr` from NumPy's generator, which
    advances its counter by one before producing a block."""
    kint = key[0] | (key[1] << 64)
    cint = sum(c << (64 * i) for i, c in enumerate(ctr))
    bg = np.random.Philox(key=kint, counter=(cint - 1) % (1 << 256))
    return bg.random_raw(4)


@pytest.mark.parametrize("key,ctr", [
    ((0, 0), (0, 0, 0, 0)),
    ((1, 0), (1, 0, 0, 0)),
    ((0x5EED, 0), (7, 3, 1, 12345)),
    ((M64, M64), (M64, M64, M64, M64)),
    ((0x0123456789ABCDEF, 0xFEDCBA9876543210), (2**63, 1, 2**40 + 17, 99)),
])
def test_philox_matches_numpy(key, ctr):
    mine = SV.philox4x64(np.array(ctr, dtype=np.uint64), key)
    np.testing.assert_array_equal(mine, _numpy_philox_block(key, ctr))


def test_philox_vectorised_counters_match_numpy():
    rng = np.random.default_rng(7)
    ctrs = rng.integers(0, 2**63, size=(16, 4), dtype=np.uint64) * np.uint64(2) + np.uint64(1)
    key = (0xDEADBEEF, 0x12345)
    mine = SV.philox4x64(ctrs, key)
    for i in range(16):
        np.testing.assert_array_equal(mine[i], _numpy_philox_block(key, [int(c) for c in ctrs[i]]))


def test_philox_words_layout():
    # word n of a stream is word n % 4 of counter (offset, request, stream, n // 4)
    seed, off, req, st = 99, 5, 3, 1
    n = np.arange(10)
    w = SV.philox_words(seed, off, req, st, n)
    for k in range(10):
        blk = _numpy_philox_block((seed, 0), (off, req, st, k // 4))
        assert w[k] == blk[k % 4]


def test_uniform_maps_end_points():
    assert SV.uniform_closed_open(np.uint64(0)) == 0.0
    assert SV.uniform_closed_open(np.uint64(M64)) == 1.0 - 2.0 ** -53
    assert SV.uniform_open(np.uint64(0)) == 2.0 ** -54
    # the top word's U' = 1 - 2^-54 is not a float64; its exponential variate
    # -ln U' is still exact and positive
    assert SV.neg_log_uniform_open(np.uint64(M64)) == pytest.approx(2.0 ** -54, rel=1e-15)
    assert SV.neg_log_uniform_open(np.uint64(0)) == pytest.approx(54 * np.log(2.0), rel=1e-15)
    # 53 significant bits: the low 11 bits of the word never matter
    assert SV.uniform_closed_open(np.uint64(2047)) == 0.0
    assert SV.uniform_closed_open(np.uint64(2048)) == 2.0 ** -53


def _neg_log_decimal(k: int) -> Decimal:
    """-ln(((k + 1/2) 2^-53)) in 50-digit decimal arithmetic."""
    with localcontext() as ctx:
        ctx.prec = 50
        u = (Decimal(k) + Decimal("0.5")) / (Decimal(2) ** 53)
        return -u.ln()


def test_neg_log_uniform_open_matches_decimal():
    # random words over both halves, the words at the switch between the two
    # formulas and the ends, against an independent 50-digit evaluation
    rng = np.random.default_rng(11)
    ks = [int(x) for x in rng.integers(0, 1 << 53, size=200, dtype=np.uint64)]
    ks += [0, 1, (1 << 52) - 1, 1 << 52, (1 << 52) + 1, (1 << 53) - 2, (1 << 53) - 1,
           (1 << 53) - 1000, 1 << 40]
    got = SV.neg_log_uniform_open(np.array(ks, dtype=np.uint64) << np.uint64(11))
    for k, g in zip(ks, got):
        want = float(_neg_log_decimal(k))
        assert g == pytest.approx(want, rel=4e-16), k


def test_streams_and_requests_are_distinct():
    a = SV.accept_uniforms(1, 0, 0, 8)
    b = SV.accept_uniforms(1, 0, 1, 8)
    c = SV.accept_uniforms(1, 1, 0, 8)
    d = SV.accept_uniforms(2, 0, 0, 8)
    for x in (b, c, d):
        assert not np.any(a == x)
    np.testing.assert_array_equal(a, SV.accept_uniforms(1, 0, 0, 8))
    u = SV.draw_uniforms(1, 0, 0, 4000)
    assert np.all((u > 0) & (u < 1))
    # roughly uniform: Kolmogorov-Smirnov against U(0, 1)
    assert scipy.stats.kstest(u, "uniform").pvalue > 1e-4


# ---------------------------------------------------------------- the theorem

P0 = np.array([0.05, 0.30, 0.10, 0.25, 0.20, 0.10])
Q1 = np.array([0.30, 0.05, 0.25, 0.10, 0.10, 0.20])


def _first_tokens(n, tau=1.0, seed=0x5EED, offset=0, p=P0, q=Q1, B=2):
    """Run n requests whose drafted d_1 is drawn from q (NumPy generator, an input),
    and return the first emitted token of each and its accept length."""
    V = len(p)
    rng = np.random.default_rng(11)
    Z = np.zeros((B, V))
    Y = np.zeros((B, V))
    Z[0] = np.log(p) * tau  # softmax(Z_0 / tau) = p
    Y[1] = np.log(q) * tau
    Z[1:] = rng.normal(size=(B - 1, V))
    Y[2:] = rng.normal(size=(B - 2, V)) if B > 2 else Y[2:]
    xs = rng.choice(V, size=n, p=q)
    first = np.empty(n, dtype=np.int64)
    acc = np.empty(n, dtype=np.int64)
    for r in range(n):
        d = [0, int(xs[r])] + [int(t) for t in rng.integers(0, V, size=B - 2)]
        res = SV.sampled_verify_request(Z, Y, d, tau, seed, offset, r)
        first[r] = res["emitted"][0]
        acc[r] = res["a"]
    return first, acc


def _chi2_pvalue(tokens, p):
    obs = np.bincount(tokens, minlength=len(p))
    return scipy.stats.chisquare(obs, len(tokens) * p).pvalue


@pytest.mark.parametrize("tau", [1.0, 0.6])
def test_first_token_is_distributed_as_target(tau):
    first, _ = _first_tokens(6000, tau=tau)
    assert _chi2_pvalue(first, P0) > 1e-4


def test_planted_mistake_fails_the_distribution_check(monkeypatch):
    # drawing the replacement from p instead of max(0, p - q) biases the output
    monkeypatch.setattr(SV, "residual_log_weights", lambda lp, lq: lp)
    first, _ = _first_tokens(4000)
    assert _chi2_pvalue(first, P0) < 1e-8


def test_acceptance_rate_is_one_minus_total_variation():
    n = 10000
    _, acc = _first_tokens(n)
    tv = 0.5 * np.abs(P0 - Q1).sum()
    rate = (acc == 1).mean()
    sd = np.sqrt((1 - tv) * tv / n)
    assert abs(rate - (1 - tv)) < 5 * sd


def test_bonus_draw_is_distributed_as_last_target_row():
    # q equal to p at every position: every draft token is accepted and the
    # drawn token follows p_{B-1}
    V, B, n = 5, 3, 6000
    pl = np.array([0.1, 0.4, 0.2, 0.2, 0.1])
    Z = np.log(np.array([[0.2] * 5, [0.1, 0.1, 0.6, 0.1, 0.1], pl]))
    Y = np.vstack([np.zeros(V), Z[0], Z[1]])
    toks = np.empty(n, dtype=np.int64)
    for r in range(n):
        res = SV.sampled_verify_request(Z, Y, [0, r % V, (3 * r) % V], 1.0, 7, 0, r)
        assert res["a"] == B - 1
        toks[r] = res["token"]
    assert _chi2_pvalue(toks, pl) > 1e-4


def test_gumbel_argmax_frequencies():
    p = np.array([0.5, 0.25, 0.125, 0.125])
    toks = [SV.gumbel_argmax(np.log(p), SV.draw_exponentials(3, 0, r, 4))[0] for r in range(8000)]
    assert _chi2_pvalue(np.array(toks), p) > 1e-4


# ---------------------------------------------------------------- limits and special cases

def test_zero_temperature_limit_is_greedy_verify():
    # with tau -> 0, p_i is a point mass at argmax Z_i and q_j one at argmax Y_j;
    # the draft proposes its own argmax, so sampled verify must equal greedy verify
    b, B, V = 6, 6, 50
    case = synth.make_verify_case(b, B, V, "sv_greedy", plant=("uniform",), dtype="f32")
    Z = case["logits"].double().numpy()
    d = case["draft"].numpy()
    Y = np.random.default_rng(3).normal(size=(b, B, V))
    for r in range(b):
        for j in range(1, B):
            Y[r, j, d[r, j]] = Y[r, j].max() + 5.0
    out = np.zeros((b, 4 * B), dtype=np.int64)
    z = np.zeros(b, dtype=np.int64)
    greedy = O.verify_batch(Z, d, out, z, 4 * B, z)
    sampled = SV.sampled_verify_batch(Z, Y, d, 1e-4, 0x5EED, 0, out, z, 4 * B, z)
    for k in ("out_tokens", "out_len", "seq_lens", "accept", "next_anchor", "status"):
        np.testing.assert_array_equal(sampled[k], greedy[k], err_msg=k)
    assert len(set(greedy["accept"].tolist())) > 1  # the case is not degenerate


def test_sure_accept_and_sure_reject():
    V, B = 8, 5
    rng = np.random.default_rng(5)
    Y = rng.normal(size=(B, V))
    d = [1, 2, 3, 4, 5]
    # target puts at least the draft's probability on every proposal: always accepted
    Z = np.vstack([Y[1:], rng.normal(size=(1, V))])
    for i in range(B - 1):
        Z[i, d[i + 1]] += 1.0
    for r in range(50):
        assert SV.sampled_verify_request(Z, Y, d, 1.0, 1, 0, r)["a"] == B - 1
    # target gives the first proposal a vanishing probability: always rejected at 0,
    # and the replacement is never the rejected token (its residual weight is 0)
    Z2 = Z.copy()
    Z2[0, d[1]] = -1e4
    for r in range(50):
        res = SV.sampled_verify_request(Z2, Y, d, 1.0, 1, 0, r)
        assert res["a"] == 0 and res["token"] != d[1]


def test_residual_log_weights_special_values():
    lp = np.log(np.array([0.5, 0.3, 0.2]))
    lq = np.log(np.array([0.25, 0.3, 0.45]))
    w = SV.residual_log_weights(lp, lq)
    np.testing.assert_allclose(np.exp(w[0]), 0.25, rtol=1e-14)
    assert w[1] == -np.inf and w[2] == -np.inf


def test_batch_bookkeeping_and_statuses():
    b, B, V = 4, 4, 32
    case = synth.make_sampled_verify_case(b, B, V, "sv_book", dtype="f32")
    Z = case["target"].double().numpy()
    Y = case["draft_logits"].double().numpy()
    d = case["draft"].numpy().astype(np.int64)
    d[2, 3] = V  # out of range: request 2 writes nothing
    out = np.full((b, 6), -1, dtype=np.int64)
    out_len = np.array([0, 3, 0, 5])  # request 3 has room for one token only
    seq = np.array([10, 20, 30, 40])
    res = SV.sampled_verify_batch(Z, Y, d, 0.8, 9, 2, out, out_len, 6, seq)
    assert res["status"][2] == SV.VERIFY_TOKEN_RANGE
    assert (res["out_tokens"][2] == -1).all() and res["out_len"][2] == 0
    for r in (0, 1):
        a = res["accept"][r]
        det = res["detail"][r]
        assert 0 <= a <= B - 1 and det["a"] == a
        assert res["out_len"][r] == out_len[r] + a + 1 and res["seq_lens"][r] == seq[r] + a + 1
        got = res["out_tokens"][r, out_len[r]:out_len[r] + a + 1].tolist()
        assert got == d[r, 1:a + 1].tolist() + [det["token"]] == det["emitted"]
        assert res["next_anchor"][r] == det["token"]
    a3 = res["detail"][3]["a"]
    if a3 + 1 > 1:
        assert res["status"][3] == SV.VERIFY_OUT_CAP and res["out_len"][3] == 5
    else:
        assert res["status"][3] == SV.VERIFY_OK and res["out_len"][3] == 6
