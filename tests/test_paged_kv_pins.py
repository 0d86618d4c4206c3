"""Pins for the paged K/V oracle (oracle/paged_kv.py).

Paging changes where a row lives, never its value, so every check reduces to
the contiguous oracle (pinned in test_oracle_pins.py):

* an identity page table over a pool that is the contiguous cache reshaped
  gives back that cache bit for bit, and the same draft;
* injection through a randomly permuted page table, gathered back, equals
  contiguous injection;
* a request that shares another request's prefix pages, and injects only its
  own suffix, drafts exactly as it does with private pages holding its whole
  injected context;
* unmapped pages are reported and leave the pools untouched.
"""

import numpy as np
import torch

import oracle as O
import synth
from tests.test_oracle_pins import MICRO, _micro_caches, micro_weights

PK = O.paged_kv
P = 4  # positions per page


def _model(B=4):
    cfg = MICRO.replace(B=B)
    return cfg, O.Weights64(micro_weights(cfg), cfg)


def _contiguous_inject(taps, cu, st, W, cfg, cap, b):
    K = np.zeros((cfg.L, b, cap, cfg.nkv, cfg.hd))
    V = np.zeros_like(K)
    rows = O.inject_kv_requests(taps, cu, st, W, cfg)
    for (l, r), (pos, k, v) in rows.items():
        K[l, r, pos] = k
        V[l, r, pos] = v
    return K, V


def test_identity_table_is_the_contiguous_cache():
    cfg, W = _model()
    T, m = 7, 2  # 7 context positions in 2 pages of 4
    caches = _micro_caches(cfg, m * P)
    K_pool = np.zeros((cfg.L, m, cfg.nkv, P, cfg.hd))
    V_pool = np.zeros_like(K_pool)
    for l, (K, V) in enumerate(caches):
        K_pool[l] = K.reshape(m, P, cfg.nkv, cfg.hd).transpose(0, 2, 1, 3)
        V_pool[l] = V.reshape(m, P, cfg.nkv, cfg.hd).transpose(0, 2, 1, 3)
    got = PK.gather_caches(K_pool, V_pool, [0, 1], T, P)
    for (Kg, Vg), (K, V) in zip(got, caches):
        np.testing.assert_array_equal(Kg, K[:T])
        np.testing.assert_array_equal(Vg, V[:T])
    toks, _ = PK.draft_block_paged(5, T, K_pool, V_pool, [0, 1], P, W, cfg, steps=2)
    want, _ = O.draft_block(5, T, [(K[:T], V[:T]) for K, V in caches], W, cfg, steps=2)
    np.testing.assert_array_equal(toks, want)


def test_permuted_pages_inject_like_contiguous():
    cfg, W = _model()
    b, cap = 3, 12
    n_pages = b * cap // P + 2  # two spare pages stay untouched
    ctx = torch.tensor([12, 9, 5], dtype=torch.int32)
    cfgb = cfg.replace(batch=b)
    cu, st, n = synth.make_inject_layout(cfgb, ctx, "prefill")
    taps = synth.make_tap_hiddens(cfgb, n, label="paged_taps")
    perm = np.random.default_rng(3).permutation(n_pages)
    table = perm[: b * cap // P].reshape(b, cap // P)
    K0 = np.full((cfg.L, n_pages, cfg.nkv, P, cfg.hd), 7.0)
    Kp, Vp, status = PK.inject_kv_paged(taps, cu, st, table, P, W, cfg, K0, K0.copy())
    assert (status == PK.STATUS_OK).all()
    Kc, Vc = _contiguous_inject(taps, cu, st, W, cfg, cap, b)
    for r in range(b):
        T = int(ctx[r])
        got = PK.gather_caches(Kp, Vp, table[r], T, P)
        for l, (Kg, Vg) in enumerate(got):
            np.testing.assert_array_equal(Kg, Kc[l, r, :T])
            np.testing.assert_array_equal(Vg, Vc[l, r, :T])
    for spare in perm[b * cap // P:]:
        assert (Kp[:, spare] == 7.0).all() and (Vp[:, spare] == 7.0).all()


def test_shared_prefix_pages_draft_like_private_pages():
    cfg, W = _model(B=4)
    prefix, T1 = 8, 11  # request 1: the 8-position prefix of request 0, then 3 of its own
    cfg1 = cfg.replace(batch=1)
    # request 0's context rows 0..9 and request 1's suffix rows 8..10 (own hidden states)
    taps0 = synth.make_tap_hiddens(cfg1, 10, label="prefix0")
    taps1s = synth.make_tap_hiddens(cfg1, T1 - prefix, label="suffix1")
    taps1 = [torch.cat([a[:prefix], s]) for a, s in zip(taps0, taps1s)]  # request 1's full context
    n_pages = 8
    # shared: pages 0, 1 hold positions 0..7 for both; request 0 owns page 2, request 1 page 3
    table = np.array([[0, 1, 2], [0, 1, 3]])
    pool = np.zeros((cfg.L, n_pages, cfg.nkv, P, cfg.hd))
    Kp, Vp, s0 = PK.inject_kv_paged(taps0, torch.tensor([0, 10]), torch.tensor([0]), table[:1], P,
                                    W, cfg, pool, pool)
    Kp, Vp, s1 = PK.inject_kv_paged(taps1s, torch.tensor([0, T1 - prefix]),
                                    torch.tensor([prefix]), table[1:], P, W, cfg, Kp, Vp)
    assert s0[0] == PK.STATUS_OK and s1[0] == PK.STATUS_OK
    # the same request with private pages 4, 5, 6 and its whole context injected
    private = np.array([[4, 5, 6]])
    Kq, Vq, s2 = PK.inject_kv_paged(taps1, torch.tensor([0, T1]), torch.tensor([0]), private, P, W,
                                    cfg, Kp, Vp)
    assert s2[0] == PK.STATUS_OK
    shared_view = PK.gather_caches(Kp, Vp, table[1], T1, P)
    private_view = PK.gather_caches(Kq, Vq, private[0], T1, P)
    for (a, b_), (c, d) in zip(shared_view, private_view):
        np.testing.assert_array_equal(a, c)
        np.testing.assert_array_equal(b_, d)
    t_sh, _ = PK.draft_block_paged(9, T1, Kp, Vp, table[1], P, W, cfg, steps=2)
    t_pr, _ = PK.draft_block_paged(9, T1, Kq, Vq, private[0], P, W, cfg, steps=2)
    np.testing.assert_array_equal(t_sh, t_pr)
    # request 0 still sees its own third page
    c0 = PK.gather_caches(Kp, Vp, table[0], 10, P)
    assert not np.array_equal(c0[0][0][8:10], shared_view[0][0][8:10])


def test_unmapped_pages_are_reported_and_write_nothing():
    cfg, W = _model()
    cfg2 = cfg.replace(batch=2)
    ctx = torch.tensor([6, 6], dtype=torch.int32)
    cu, st, n = synth.make_inject_layout(cfg2, ctx, "prefill")
    taps = synth.make_tap_hiddens(cfg2, n, label="paged_bad")
    table = np.array([[0, 1], [2, -1]])  # request 1's positions 4, 5 have no page
    pool = np.zeros((cfg.L, 3, cfg.nkv, P, cfg.hd))
    Kp, Vp, status = PK.inject_kv_paged(taps, cu, st, table, P, W, cfg, pool, pool)
    assert list(status) == [PK.STATUS_OK, PK.STATUS_PAGE]
    assert (Kp[:, 2] == 0).all() and (Vp[:, 2] == 0).all()  # request 1 wrote nothing
    assert np.abs(Kp[:, :2]).max() > 0
    assert PK.gather_caches(Kp, Vp, table[1], 6, P) is None
    assert PK.gather_caches(Kp, Vp, [0, 9], 6, P) is None  # id outside the pool
    assert PK.draft_block_paged(1, 6, Kp, Vp, table[1], P, W, cfg) == (None, None)
