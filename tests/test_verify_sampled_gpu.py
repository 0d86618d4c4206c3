"""Sampled verify on the GPU against the oracle (oracle/sampled_verify.py).

Both sides draw the same Philox4x64-10 uniforms, so every decision has one
right answer.  The kernel takes those decisions in fp32 and the oracle in
float64, so a decision whose margin is below BAND may go either way:

* an accept decision with |log rho_i - log U_i| < BAND;
* a draw whose winning Gumbel score is within BAND of the runner-up.

Such cases are counted.  When the accept length differs, the oracle is
teacher-forced to the GPU's length and its draw is recomputed there.
Everything else must match exactly: the accept lengths, the emitted tokens,
the drawn token, the out_len / seq_lens / next_anchor bookkeeping, the error
bits and the untouched requests.
"""

import numpy as np
import pytest
import scipy.stats
import torch

import oracle as O
import synth
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu

SV = O.sampled_verify
BAND = 1e-3


def _run(Z, Y, d, tau, seed, offset, out, out_len, seq, ws=None):
    b, B, V = Z.shape
    g = {k: v.cuda() for k, v in dict(Z=Z, Y=Y, d=d, out=out, out_len=out_len, seq=seq).items()}
    acc = torch.full((b,), -9, dtype=torch.int32, device="cuda")
    nxt = torch.full((b,), -9, dtype=torch.int32, device="cuda")
    if ws is None:
        ws = D.new_workspace(D.verify_sampled_workspace_size(b, B, V))
    D.verify_sampled(g["Z"], g["Y"], g["d"], tau, seed, offset, g["out"], g["out_len"], g["seq"],
                     acc, nxt, ws)
    torch.cuda.synchronize()
    return {"out_tokens": g["out"].cpu().numpy(), "out_len": g["out_len"].cpu().numpy(),
            "seq_lens": g["seq"].cpu().numpy(), "accept": acc.cpu().numpy(),
            "next_anchor": nxt.cpu().numpy(), "err": D.get_error(ws)}


def _decisions(Zr, Yr, dr, tau, seed, offset, r):
    """Oracle log rho_i - log U_i for every i (positive = accept)."""
    B = Zr.shape[0]
    lp = SV.log_softmax(Zr, tau)
    lq = SV.log_softmax(Yr, tau)
    U = SV.accept_uniforms(seed, offset, r, B - 1)
    out = []
    for i in range(B - 1):
        x = int(dr[i + 1])
        lu = np.log(U[i]) if U[i] > 0 else -np.inf
        out.append(float(lp[i, x] - lq[i + 1, x] - lu))
    return np.array(out), lp, lq


def _draw_at(lp, lq, a, B, seed, offset, r, V):
    logw = SV.residual_log_weights(lp[a], lq[a + 1]) if a < B - 1 else lp[B - 1]
    if not np.any(np.isfinite(logw)):
        logw = lp[a]
    return SV.gumbel_argmax(logw, SV.draw_exponentials(seed, offset, r, V))


def _check(Z, Y, d, tau, seed, offset, out0, ol0, seq0, res, stats):
    """Per request: accept length within the near-tie rule, drawn token within the
    score band, and exact bookkeeping."""
    Zd, Yd = Z.double().numpy(), Y.double().numpy()
    dn = d.numpy().astype(np.int64)
    b, B, V = Zd.shape
    cap = out0.shape[1]
    for r in range(b):
        marg, lp, lq = _decisions(Zd[r], Yd[r], dn[r], tau, seed, offset, r)
        a_or = int(np.argmax(marg <= 0)) if np.any(marg <= 0) else B - 1
        a = int(res["accept"][r])
        assert 0 <= a <= B - 1, r
        # the GPU's length must be one the oracle admits: every earlier decision an
        # accept (margin > 0) or a near-tie, the stopping one a reject or a near-tie
        assert np.all(marg[:a] > -BAND), (r, a, a_or, marg)
        assert a == B - 1 or marg[a] < BAND, (r, a, a_or, marg)
        if a != a_or:
            stats["accept_near_ties"] += 1
        tok_or, score = _draw_at(lp, lq, a, B, seed, offset, r, V)
        tok = int(res["next_anchor"][r])
        if tok != tok_or:
            assert np.isfinite(score[tok]) and score[tok] >= score[tok_or] - BAND, (r, tok, tok_or)
            stats["draw_near_ties"] += 1
        stats["requests"] += 1
        ol = int(ol0[r])
        emitted = dn[r, 1:a + 1].tolist() + [tok]
        assert res["out_tokens"][r, ol:ol + a + 1].tolist() == emitted, r
        assert (res["out_tokens"][r, :ol] == out0[r, :ol].numpy()).all()
        assert (res["out_tokens"][r, ol + a + 1:cap] == out0[r, ol + a + 1:cap].numpy()).all()
        assert res["out_len"][r] == ol + a + 1 and res["seq_lens"][r] == int(seq0[r]) + a + 1


def _case(b, B, V, label, dtype="bf16", plant=("geometric", 4.0)):
    c = synth.make_sampled_verify_case(b, B, V, label, plant=plant, dtype=dtype)
    cap = 3 * B
    out0 = torch.full((b, cap), -1, dtype=torch.int32)
    ol0 = torch.randint(0, B + 1, (b,), generator=torch.Generator().manual_seed(b * B), dtype=torch.int32)
    seq0 = torch.randint(100, 5000, (b,), generator=torch.Generator().manual_seed(V), dtype=torch.int32)
    return c, out0, ol0, seq0


@pytest.mark.parametrize("b,B,V,dtype", [
    (8, 8, 20000, "bf16"),     # several chunks per row
    (8, 8, 20000, "f32"),
    (5, 4, 1001, "bf16"),      # odd vocabulary: no 16-byte rows
    (3, 16, 4099, "f32"),
    (64, 2, 3000, "bf16"),
    (2, 32, 777, "bf16"),      # a full warp of rows
    (300, 4, 2048, "bf16"),    # balanced stats CTAs span several rows and requests
])
@pytest.mark.parametrize("tau", [0.3, 1.0, 2.5])
def test_sampled_verify_matches_oracle(b, B, V, dtype, tau):
    c, out0, ol0, seq0 = _case(b, B, V, f"sv_{b}_{B}_{V}", dtype=dtype)
    seed, offset = 0x5EED + b, 7 * B
    res = _run(c["target"], c["draft_logits"], c["draft"], tau, seed, offset, out0, ol0, seq0)
    assert res["err"] == 0
    stats = dict(requests=0, accept_near_ties=0, draw_near_ties=0)
    _check(c["target"], c["draft_logits"], c["draft"], tau, seed, offset, out0, ol0, seq0, res,
           stats)
    print(stats)
    assert stats["accept_near_ties"] + stats["draw_near_ties"] <= max(1, b // 8)


def test_sampled_verify_full_size_8b_bs32():
    b, B, V = 32, 8, 151936
    c, out0, ol0, seq0 = _case(b, B, V, "sv_full")
    res = _run(c["target"], c["draft_logits"], c["draft"], 1.0, 12345, 99, out0, ol0, seq0)
    assert res["err"] == 0
    stats = dict(requests=0, accept_near_ties=0, draw_near_ties=0)
    _check(c["target"], c["draft_logits"], c["draft"], 1.0, 12345, 99, out0, ol0, seq0, res, stats)
    print(stats)
    a = res["accept"]
    assert len(set(a.tolist())) > 2  # planted prefixes give a spread of accept lengths


def test_sampled_verify_repeats_with_equal_seed_and_offset():
    c, out0, ol0, seq0 = _case(16, 8, 5000, "sv_rep")
    args = (c["target"], c["draft_logits"], c["draft"], 0.8)
    r1 = _run(*args, 1, 2, out0, ol0, seq0)
    r2 = _run(*args, 1, 2, out0, ol0, seq0)
    for k in ("out_tokens", "out_len", "seq_lens", "accept", "next_anchor"):
        assert np.array_equal(r1[k], r2[k]), k
    r3 = _run(*args, 1, 3, out0, ol0, seq0)
    assert not np.array_equal(r1["next_anchor"], r3["next_anchor"])


def test_sampled_verify_first_token_follows_target_distribution():
    # the speculative-sampling theorem through the GPU path: d_1 drawn from q
    # (an input drawn with NumPy), first emitted token ~ p_0
    n, V, tau = 6000, 6, 1.0
    p = np.array([0.05, 0.30, 0.10, 0.25, 0.20, 0.10])
    q = np.array([0.30, 0.05, 0.25, 0.10, 0.10, 0.20])
    Z = torch.zeros((n, 2, V), dtype=torch.float32)
    Y = torch.zeros((n, 2, V), dtype=torch.float32)
    Z[:, 0] = torch.tensor(np.log(p), dtype=torch.float32)
    Y[:, 1] = torch.tensor(np.log(q), dtype=torch.float32)
    xs = np.random.default_rng(11).choice(V, size=n, p=q)
    d = torch.zeros((n, 2), dtype=torch.int32)
    d[:, 1] = torch.tensor(xs, dtype=torch.int32)
    out0 = torch.full((n, 2), -1, dtype=torch.int32)
    z = torch.zeros(n, dtype=torch.int32)
    res = _run(Z, Y, d, tau, 0xC0FFEE, 0, out0, z, z)
    assert res["err"] == 0
    first = res["out_tokens"][:, 0]
    obs = np.bincount(first, minlength=V)
    assert scipy.stats.chisquare(obs, n * p).pvalue > 1e-4
    tv = 0.5 * np.abs(p - q).sum()
    rate = (res["accept"] == 1).mean()
    assert abs(rate - (1 - tv)) < 5 * np.sqrt(tv * (1 - tv) / n)


def test_sampled_verify_errors_write_nothing():
    b, B, V = 4, 4, 2000
    c, out0, ol0, seq0 = _case(b, B, V, "sv_err")
    d = c["draft"].clone()
    d[1, 2] = V          # token out of range: request 1 untouched
    ol0 = ol0.clone()
    ol0[3] = 3 * B - 1   # room for one token: request 3 overflows unless a == 0
    res = _run(c["target"], c["draft_logits"], d, 1.0, 5, 0, out0, ol0, seq0)
    assert res["err"] & D.DEV_TOKEN_RANGE
    assert (res["out_tokens"][1] == -1).all()
    assert res["out_len"][1] == ol0[1] and res["seq_lens"][1] == seq0[1]
    assert res["accept"][1] == -9 and res["next_anchor"][1] == -9
    if res["accept"][3] == -9:
        assert res["err"] & D.DEV_OUT_CAP and res["out_len"][3] == ol0[3]
    # the other requests are unaffected
    for r in (0, 2):
        assert 0 <= res["accept"][r] <= B - 1


def test_sampled_verify_workspace_reuse():
    b, B, V = 6, 8, 3000
    c, out0, ol0, seq0 = _case(b, B, V, "sv_ws")
    ws = D.new_workspace(max(D.verify_sampled_workspace_size(b, B, V),
                             D.verify_workspace_size(b, B, V)))
    first = _run(c["target"], c["draft_logits"], c["draft"], 1.0, 9, 1, out0, ol0, seq0, ws=ws)
    # a greedy verify in between uses the same counters
    g = synth.make_verify_case(b, B, V, "sv_ws_greedy")
    acc = torch.zeros(b, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(b, dtype=torch.int32, device="cuda")
    D.verify(g["logits"].cuda(), g["draft"].cuda(), out0.clone().cuda(), ol0.clone().cuda(),
             seq0.clone().cuda(), acc, nxt, ws)
    again = _run(c["target"], c["draft_logits"], c["draft"], 1.0, 9, 1, out0, ol0, seq0, ws=ws)
    for k in ("out_tokens", "out_len", "seq_lens", "accept", "next_anchor"):
        assert np.array_equal(first[k], again[k]), k
    assert first["err"] == 0 and again["err"] == 0
