"""Pins for the fp64 oracle: closed forms, invariants and a brute-force twin.

None of these re-types the oracle's formulas against themselves: each check is
a closed-form value, a mathematical invariant, an independent library routine
(scipy's softmax) or the loop-based restatement in ``tests/bruteforce.py``.
"""

import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
import synth
from synth.configs import DraftConfig
from tests import bruteforce as BF

MICRO = DraftConfig(
    name="micro", dtype="f32", H_t=4, n_tap=2, L=2, d=8, nq=4, nkv=2, hd=4, I=8, V=16,
    batch=2, ctx=("fixed", 3), B=3, steps=1, plant=("uniform",), eps=1e-6, rope_base=100.0,
    w_std=0.5, h_std=1.0, gain_std=0.3)


def micro_weights(cfg=MICRO):
    return synth.make_weights(cfg)


def nested(t):
    return t.double().tolist()


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_form():
    x = np.array([3.0, 4.0])
    r = math.sqrt((9 + 16) / 2)
    np.testing.assert_allclose(O.rms_norm(x, [1.0, 1.0], 0.0), [3 / r, 4 / r], rtol=1e-15)
    np.testing.assert_allclose(O.rms_norm(x, [2.0, 0.5], 0.0), [6 / r, 2 / r], rtol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 64))
    y = O.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, np.ones(64), 0.0), y, rtol=1e-13)
    # eps enters under the root: a zero row stays zero, a tiny row is damped
    z = O.rms_norm(np.full((1, 4), 1e-4), np.ones(4), 1e-6)
    np.testing.assert_allclose(z, 1e-4 / math.sqrt(1e-8 + 1e-6), rtol=1e-14)


# ---------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    x = np.random.default_rng(1).normal(size=(3, 2, 8))
    np.testing.assert_array_equal(O.apply_rope(x, [0, 0, 0], 1e6), x)


def test_rope_closed_form_rotation():
    # hd = 2: one pair, theta_0 = 1 -> (1, 0) at position p becomes (cos p, sin p)
    for p in (1, 2, 5, 100):
        y = O.apply_rope(np.array([[[1.0, 0.0]]]), [p], 1e6)
        np.testing.assert_allclose(y[0, 0], [math.cos(p), math.sin(p)], rtol=1e-14, atol=1e-14)
    # hd = 4, base 100: theta_1 = 100^(-1/2) = 0.1; pair (1, 3) turns by 0.1 p
    x = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    y = O.apply_rope(x, [7], 100.0)
    np.testing.assert_allclose(y[0, 0], [0.0, math.cos(0.7), 0.0, math.sin(0.7)], atol=1e-14)


def test_rope_preserves_norm_and_depends_on_relative_position():
    rng = np.random.default_rng(2)
    q = rng.normal(size=(1, 1, 16))
    k = rng.normal(size=(1, 1, 16))
    for p in (3, 77, 4095, 32768):
        np.testing.assert_allclose(np.linalg.norm(O.apply_rope(q, [p], 1e6)), np.linalg.norm(q),
                                   rtol=1e-13)
    dots = []
    for m, n in ((10, 4), (106, 100), (32774, 32768)):
        dots.append(float((O.apply_rope(q, [m], 1e6) * O.apply_rope(k, [n], 1e6)).sum()))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


def test_silu_closed_form():
    np.testing.assert_allclose(O.silu(np.array([0.0, 1.0, -2.0])),
                               [0.0, 1 / (1 + math.exp(-1)), -2 / (1 + math.exp(2))], rtol=1e-15)


# ---------------------------------------------------------------- attention

def _loop_attention(q, K, V):
    B, nq, hd = q.shape
    grp = nq // K.shape[1]
    o = np.zeros_like(q)
    for j in range(B):
        for a in range(nq):
            sc = [sum(q[j, a, e] * K[t, a // grp, e] for e in range(hd)) / math.sqrt(hd)
                  for t in range(K.shape[0])]
            m = max(sc)
            w = [math.exp(s - m) for s in sc]
            for e in range(hd):
                o[j, a, e] = sum(w[t] * V[t, a // grp, e] for t in range(len(w))) / sum(w)
    return o


def test_block_attention_matches_loops():
    rng = np.random.default_rng(3)
    q = rng.normal(size=(3, 4, 4))
    Kc, Vc = rng.normal(size=(5, 2, 4)), rng.normal(size=(5, 2, 4))
    kb, vb = rng.normal(size=(3, 2, 4)), rng.normal(size=(3, 2, 4))
    got = O.block_attention(q, Kc, Vc, kb, vb)
    want = _loop_attention(q, np.concatenate([Kc, kb]), np.concatenate([Vc, vb]))
    np.testing.assert_allclose(got, want, rtol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(4)
    q = rng.normal(size=(4, 8, 16))
    Kc, Vc = rng.normal(size=(9, 2, 16)), rng.normal(size=(9, 2, 16))
    kb, vb = rng.normal(size=(4, 2, 16)), rng.normal(size=(4, 2, 16))
    rep = lambda a: np.repeat(a, 4, axis=1)
    np.testing.assert_allclose(O.block_attention(q, Kc, Vc, kb, vb),
                               O.block_attention(q, rep(Kc), rep(Vc), rep(kb), rep(vb)), rtol=1e-13)


def test_attention_equal_keys_average_values():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(2, 2, 4))
    K = np.ones((6, 1, 4))
    V = rng.normal(size=(6, 1, 4))
    o = O.block_attention(q, K[:4], V[:4], K[4:], V[4:])
    np.testing.assert_allclose(o, np.broadcast_to(V.mean(0)[None], o.shape), rtol=1e-13)


def test_attention_empty_context():
    rng = np.random.default_rng(6)
    q = rng.normal(size=(3, 2, 4))
    kb, vb = rng.normal(size=(3, 1, 4)), rng.normal(size=(3, 1, 4))
    got = O.block_attention(q, np.zeros((0, 1, 4)), np.zeros((0, 1, 4)), kb, vb)
    np.testing.assert_allclose(got, _loop_attention(q, kb, vb), rtol=1e-12)


# ---------------------------------------------------------------- context features / injection

def test_context_features_scalar_closed_form():
    # H_t = 1, two taps, d = 1: u = h1 w1 + h2 w2 and RMSNorm of a scalar is sign(u) * g
    taps = [np.array([[2.0], [-1.0]]), np.array([[0.5], [3.0]])]
    W = np.array([[1.5, -4.0]])
    c = O.context_features(taps, W, np.array([0.7]), 0.0)
    np.testing.assert_allclose(c[:, 0], [np.sign(3 - 2) * 0.7, np.sign(-1.5 - 12) * 0.7])


def test_context_features_tap_order_is_ascending():
    # W_fc picks tap 0 into output 0 and tap 1 into output 1
    taps = [np.array([[1.0]]), np.array([[3.0]])]
    c = O.context_features(taps, np.eye(2), np.ones(2), 0.0)
    r = math.sqrt((1 + 9) / 2)
    np.testing.assert_allclose(c[0], [1 / r, 3 / r], rtol=1e-15)


def test_inject_matches_bruteforce_and_chunking():
    cfg = MICRO
    w = micro_weights()
    W = O.Weights64(w, cfg)
    taps = synth.make_tap_hiddens(cfg, 7)
    cu = torch.tensor([0, 3, 7], dtype=torch.int32)
    st = torch.tensor([0, 5], dtype=torch.int32)
    full = O.inject_kv_requests(taps, cu, st, W, cfg)
    # brute force, row by row
    for r, (lo, hi) in enumerate(((0, 3), (3, 7))):
        for l in range(cfg.L):
            pos, K, V = full[(l, r)]
            for i, row in enumerate(range(lo, hi)):
                c = BF.features([nested(t[row]) for t in taps], nested(w["W_fc"]),
                                nested(w["g_ctx"]), cfg.eps)
                Kb, Vb = BF.inject_row(c, int(st[r]) + i, nested(w["layers"][l]["Wk"]),
                                       nested(w["layers"][l]["Wv"]), cfg.nkv, cfg.hd, cfg.rope_base)
                np.testing.assert_allclose(K[i], Kb, rtol=1e-11, atol=1e-13)
                np.testing.assert_allclose(V[i], Vb, rtol=1e-11, atol=1e-13)
    # the second request injected in two calls (rows 3..4 then 5..6) equals one call
    a = O.inject_kv_requests([t[3:5] for t in taps], torch.tensor([0, 2]), torch.tensor([5]), W, cfg)
    b = O.inject_kv_requests([t[5:7] for t in taps], torch.tensor([0, 2]), torch.tensor([7]), W, cfg)
    for l in range(cfg.L):
        np.testing.assert_array_equal(np.concatenate([a[(l, 0)][1], b[(l, 0)][1]]), full[(l, 1)][1])
        np.testing.assert_array_equal(np.concatenate([a[(l, 0)][2], b[(l, 0)][2]]), full[(l, 1)][2])


def test_inject_position_moves_k_not_v():
    cfg = MICRO
    W = O.Weights64(micro_weights(), cfg)
    taps = synth.make_tap_hiddens(cfg, 1)
    one = torch.tensor([0, 1])
    x = O.inject_kv_requests(taps, one, torch.tensor([0]), W, cfg)
    y = O.inject_kv_requests(taps, one, torch.tensor([9]), W, cfg)
    np.testing.assert_array_equal(x[(0, 0)][2], y[(0, 0)][2])
    assert np.abs(x[(0, 0)][1] - y[(0, 0)][1]).max() > 1e-3
    np.testing.assert_allclose(np.linalg.norm(x[(0, 0)][1]), np.linalg.norm(y[(0, 0)][1]), rtol=1e-13)


# ---------------------------------------------------------------- draft forward

def _micro_caches(cfg, T, seed=11):
    rng = np.random.default_rng(seed)
    return [(rng.normal(size=(T, cfg.nkv, cfg.hd)), rng.normal(size=(T, cfg.nkv, cfg.hd)))
            for _ in range(cfg.L)]


def test_draft_forward_matches_bruteforce():
    cfg = MICRO
    w = micro_weights()
    W = O.Weights64(w, cfg)
    T = 3
    caches = _micro_caches(cfg, T)
    toks = [5, cfg.mask_id, 2]
    z = O.draft_hidden(toks, T, caches, W, cfg)
    got = W.lm_logits(z)
    bf_caches = [(K.tolist(), V.tolist()) for K, V in caches]
    wn = {"emb": nested(w["emb"]), "g_final": nested(w["g_final"]), "W_lm": nested(w["W_lm"]),
          "layers": [{k: nested(v) for k, v in lw.items()} for lw in w["layers"]]}
    want = BF.forward_logits(toks, T, bf_caches, wn, cfg)
    np.testing.assert_allclose(got, np.array(want), rtol=1e-10, atol=1e-12)


def test_block_is_bidirectional():
    cfg = MICRO
    W = O.Weights64(micro_weights(), cfg)
    caches = _micro_caches(cfg, 3)
    z1 = O.draft_hidden([5, 1, 2], 3, caches, W, cfg)
    z2 = O.draft_hidden([5, 1, 9], 3, caches, W, cfg)  # change the LAST block token
    assert np.abs(z1[0] - z2[0]).max() > 1e-6  # an earlier position sees it: no causal mask
    # and the context matters
    z3 = O.draft_hidden([5, 1, 2], 3, _micro_caches(cfg, 3, seed=12), W, cfg)
    assert np.abs(z1 - z3).max() > 1e-6


def test_lm_head_stats_against_scipy_softmax():
    cfg = MICRO
    W = O.Weights64(micro_weights(), cfg)
    z = np.random.default_rng(7).normal(size=(4, cfg.d))
    st = O.lm_head_stats(z, W, keep_logits=True)
    p = scipy.special.softmax(st["logits"], axis=1)
    np.testing.assert_allclose(st["conf"], p.max(axis=1), rtol=1e-13)
    np.testing.assert_array_equal(st["tok"], p.argmax(axis=1))
    srt = np.sort(st["logits"], axis=1)
    np.testing.assert_allclose(st["margin"], srt[:, -1] - srt[:, -2], rtol=1e-13)


def test_lm_head_stats_equal_logits():
    cfg = MICRO.replace(d=2)
    w = {"W_lm": torch.zeros(16, 2)}
    st = O.lm_head_stats(np.ones((1, 2)), O.Weights64(w, cfg))
    assert st["tok"][0] == 0 and st["margin"][0] == 0.0
    np.testing.assert_allclose(st["conf"], 1.0 / 16, rtol=1e-15)
    assert list(st["cand"][0]) == list(range(16))


# ---------------------------------------------------------------- denoising schedule

@pytest.mark.parametrize("B", [2, 4, 8, 16])
def test_commit_schedule_sums_to_block(B):
    for s in range(1, B):
        rem, ks = B - 1, []
        for t in range(s):
            k = O.commit_count(rem, s - t)
            ks.append(k)
            rem -= k
        assert sum(ks) == B - 1 and rem == 0 and all(k >= 1 for k in ks)
        if s == 1:
            assert ks == [B - 1]
        if s == B - 1:
            assert ks == [1] * (B - 1)
    assert O.commit_count(7, 2) == 4 and O.commit_count(3, 1) == 3


def test_select_commits_most_confident_ties_lower_position():
    assert O.select_commits([1, 2, 3, 4], [0.1, 0.4, 0.3, 0.2], 2) == [2, 3]
    assert O.select_commits([1, 2, 3, 4], [0.5, 0.5, 0.5, 0.1], 2) == [1, 2]
    assert O.select_commits([3, 5, 6], [0.2, 0.9, 0.2], 2) == [3, 5]


def test_valid_commit_sets_band():
    pos, conf = [1, 2, 3, 4], [0.50, 0.40, 0.39, 0.10]
    sets = O.valid_commit_sets(pos, conf, 2, 0.05)
    assert [1, 2] in sets and [1, 3] in sets and len(sets) == 2
    assert O.valid_commit_sets(pos, conf, 2, 0.0) == [[1, 2]]
    assert O.valid_commit_sets(pos, conf, 4, 0.05) == [[1, 2, 3, 4]]


def test_draft_block_single_step_is_per_position_argmax():
    cfg = MICRO.replace(B=4)
    w = micro_weights(cfg)
    W = O.Weights64(w, cfg)
    caches = _micro_caches(cfg, 3)
    toks, rec = O.draft_block(7, 3, caches, W, cfg, steps=1)
    z = O.draft_hidden([7] + [cfg.mask_id] * 3, 3, caches, W, cfg)
    want = [BF.argmax_first(row) for row in W.lm_logits(z).tolist()]
    assert list(toks) == [7] + want[1:]
    assert rec[0]["commit"] == [1, 2, 3]


def test_draft_block_one_commit_per_step_when_steps_is_block_minus_one():
    cfg = MICRO.replace(B=4)
    W = O.Weights64(micro_weights(cfg), cfg)
    caches = _micro_caches(cfg, 3)
    toks, rec = O.draft_block(7, 3, caches, W, cfg, steps=3)
    assert [len(r["commit"]) for r in rec] == [1, 1, 1]
    committed = sorted(p for r in rec for p in r["commit"])
    assert committed == [1, 2, 3]
    # each position holds the argmax that its committing step computed for it (the
    # argmax is not restricted, so [MASK] itself may legitimately be drafted)
    for r in rec:
        idx = {p: i for i, p in enumerate(r["stats"]["pos"])}
        for p in r["commit"]:
            assert int(toks[p]) == int(r["stats"]["tok"][idx[p]])
    # the first commit is the most confident position of the all-mask forward
    st0 = rec[0]["stats"]
    best = st0["pos"][int(np.argmax(st0["conf"]))]
    assert rec[0]["commit"] == [best]
    # later steps see the committed token: their forward differs from the all-mask one
    z_all_mask = O.draft_hidden([7] + [cfg.mask_id] * 3, 3, caches, W, cfg)
    later = rec[1]["stats"]
    st_again = O.lm_head_stats(z_all_mask[later["pos"]], W)
    assert np.abs(st_again["conf"] - later["conf"]).max() > 0


# ---------------------------------------------------------------- verify

def test_verify_hand_example():
    # B = 4, V = 5; target argmax per row = [2, 3, 0, 4]
    L = np.full((4, 5), -1.0)
    for i, g in enumerate([2, 3, 0, 4]):
        L[i, g] = 1.0
    a, em, bonus, g = O.verify_request(L, [9, 2, 3, 1])
    assert (a, em, bonus) == (2, [2, 3, 0], 0)
    a, em, bonus, _ = O.verify_request(L, [9, 2, 3, 0])  # all match
    assert (a, em, bonus) == (3, [2, 3, 0, 4], 4)
    a, em, bonus, _ = O.verify_request(L, [9, 1, 3, 0])  # first position mismatches
    assert (a, em, bonus) == (0, [2], 2)


def test_verify_ties_go_to_lowest_index_and_ulps_decide():
    L = np.zeros((2, 6))
    L[0, [1, 3]] = 2.0               # exact tie -> 1
    one = torch.tensor([1.0], dtype=torch.bfloat16)
    up = (one.view(torch.int16) + 1).view(torch.bfloat16)
    L[1, 4] = float(one)
    L[1, 2] = float(up)              # one bf16 ulp above -> 2
    g = O.row_argmax(L)
    assert list(g) == [1, 2]


def test_verify_matches_bruteforce_prefixes():
    rng = np.random.default_rng(8)
    for _ in range(300):
        B, V = int(rng.integers(2, 9)), int(rng.integers(2, 5))
        L = rng.integers(0, 3, size=(B, V)).astype(float)  # many ties
        d = rng.integers(0, V, size=B)
        a, em, bonus, g = O.verify_request(L, d)
        gb = [BF.argmax_first(list(r)) for r in L]
        assert list(g) == gb
        assert a == BF.accept_all_prefixes(gb, list(d))
        assert 0 <= a <= B - 1 and len(em) == a + 1 and em[-1] == gb[a]
        assert em[:a] == [int(t) for t in d[1:a + 1]]


@pytest.mark.parametrize("B", [4, 8, 16])
def test_verify_planted_cases(B):
    V = 1000
    case = synth.make_verify_case(8, B, V, "pin", plant=("uniform",))
    r = O.verify_batch(case["logits"], case["draft"], np.zeros((8, 64)), np.zeros(8), 64,
                       np.full(8, 100))
    assert np.array_equal(r["accept"], case["planted"].numpy())
    assert np.array_equal(r["out_len"], r["accept"] + 1)
    assert np.array_equal(r["seq_lens"], 100 + r["accept"] + 1)
    # all-matching drafts give B-1; a forced first-position mismatch gives 0
    L = O.as_f64(case["logits"][0])
    g = O.row_argmax(L)
    d_all = np.concatenate([[5], g[:B - 1]])
    assert O.verify_request(L, d_all)[0] == B - 1
    d_bad = d_all.copy()
    d_bad[1] = (g[0] + 1) % V
    assert O.verify_request(L, d_bad)[0] == 0


def test_verify_capacity_and_range_errors_write_nothing():
    case = synth.make_verify_case(3, 4, 50, "err")
    d = case["draft"].clone()
    d[2, 1] = 50  # outside the vocabulary
    out0 = np.full((3, 4), -7)
    r = O.verify_batch(case["logits"], d, out0, np.array([0, 3, 0]), 4, np.array([10, 10, 10]))
    assert r["status"][2] == O.VERIFY_TOKEN_RANGE and r["accept"][2] == -1
    a1 = O.verify_request(case["logits"][1], d[1])[0]
    if a1 + 1 > 1:  # 3 + a1 + 1 > 4 overflows
        assert r["status"][1] == O.VERIFY_OUT_CAP
        assert list(r["out_tokens"][1]) == [-7] * 4 and r["seq_lens"][1] == 10
    assert r["status"][0] == O.VERIFY_OK and r["out_len"][0] == r["accept"][0] + 1


# ---------------------------------------------------------------- multi-step drafting, brute force

def _bf_weights(w):
    return {"emb": nested(w["emb"]), "g_final": nested(w["g_final"]), "W_lm": nested(w["W_lm"]),
            "layers": [{k: nested(v) for k, v in lw.items()} for lw in w["layers"]]}


def _bf_draft(anchor, T, bf_caches, wn, cfg, steps):
    """Denoising by hand on the loop-based forward: every step reruns the whole block
    with the tokens committed so far, scores each still-masked position by its
    softmax max-probability, and commits the ceil(remaining / steps left) best
    (ties to the lower position) to their argmax.  Returns the tokens and, per
    step, (committed positions, {position: argmax of that step})."""
    B = cfg.B
    toks = [anchor] + [cfg.mask_id] * (B - 1)
    masked = list(range(1, B))
    steps_log = []
    for t in range(steps):
        logits = BF.forward_logits(toks, T, bf_caches, wn, cfg)
        score = {}
        for p in masked:
            row = logits[p]
            mx = max(row)
            score[p] = (1.0 / sum(math.exp(v - mx) for v in row), BF.argmax_first(row))
        left = steps - t
        k = (len(masked) + left - 1) // left
        ranked = sorted(masked, key=lambda p: (-score[p][0], p))
        commit = sorted(ranked[:k])
        for p in commit:
            toks[p] = score[p][1]
        steps_log.append((commit, {p: score[p][1] for p in masked}))
        masked = [p for p in masked if p not in commit]
    return toks, steps_log


@pytest.mark.parametrize("steps", [2, 3])
def test_multi_step_draft_matches_bruteforce(steps):
    cfg = MICRO.replace(B=4)
    w = micro_weights(cfg)
    W = O.Weights64(w, cfg)
    wn = _bf_weights(w)
    T = 3
    saw_changed_argmax = False
    for anchor, seed in ((7, 11), (3, 12), (12, 13), (0, 14)):
        caches = _micro_caches(cfg, T, seed=seed)
        bf_caches = [(K.tolist(), V.tolist()) for K, V in caches]
        want, log = _bf_draft(anchor, T, bf_caches, wn, cfg, steps)
        got, rec = O.draft_block(anchor, T, caches, W, cfg, steps=steps)
        assert [int(v) for v in got] == want
        assert [r["commit"] for r in rec] == [c for c, _ in log]
        # a later step re-predicts the positions still masked: somewhere its argmax
        # differs from the first step's, so committing a stale argmax would fail here
        for t in range(1, steps):
            for p, tok in log[t][1].items():
                saw_changed_argmax |= tok != log[0][1][p]
    assert saw_changed_argmax
