"""Greedy verify on the GPU against the oracle: bit-exact accept lengths,
emitted tokens, out_len / seq_lens / next_anchor updates and error handling."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def _run(logits, draft, out_tokens, out_len, seq_lens, ws=None):
    b, B, V = logits.shape
    dev = {k: v.cuda() for k, v in dict(logits=logits, draft=draft, out=out_tokens,
                                        out_len=out_len, seq=seq_lens).items()}
    acc = torch.full((b,), -9, dtype=torch.int32, device="cuda")
    nxt = torch.full((b,), -9, dtype=torch.int32, device="cuda")
    if ws is None:
        ws = D.new_workspace(D.verify_workspace_size(b, B, V))
    D.verify(dev["logits"], dev["draft"], dev["out"], dev["out_len"], dev["seq"], acc, nxt, ws)
    torch.cuda.synchronize()
    err = D.get_error(ws)
    return {"out_tokens": dev["out"].cpu(), "out_len": dev["out_len"].cpu(),
            "seq_lens": dev["seq"].cpu(), "accept": acc.cpu(), "next_anchor": nxt.cpu(),
            "err": err}


def _compare(res, want, skip_mask=None):
    b = res["accept"].shape[0]
    for r in range(b):
        if want["status"][r] != O.VERIFY_OK:
            continue
        assert int(res["accept"][r]) == want["accept"][r], r
        assert int(res["next_anchor"][r]) == want["next_anchor"][r], r
    assert np.array_equal(res["out_tokens"].numpy(), want["out_tokens"])
    assert np.array_equal(res["out_len"].numpy(), want["out_len"])
    assert np.array_equal(res["seq_lens"].numpy(), want["seq_lens"])


@pytest.mark.parametrize("b", synth.VERIFY_SWEEP["batches"])
@pytest.mark.parametrize("B", synth.VERIFY_SWEEP["blocks"])
def test_verify_sweep_bit_exact(b, B):
    V = synth.VERIFY_SWEEP["V"]
    case = synth.make_verify_case(b, B, V, "sweep", plant=("uniform",), adversarial=True)
    cap = 3 * B
    out0 = torch.full((b, cap), -1, dtype=torch.int32)
    ol0 = torch.zeros(b, dtype=torch.int32)
    seq0 = torch.randint(100, 5000, (b,), dtype=torch.int32)
    res = _run(case["logits"], case["draft"], out0, ol0, seq0)
    want = O.verify_batch(case["logits"], case["draft"], out0, ol0, cap, seq0)
    assert res["err"] == 0
    assert (want["status"] == 0).all()
    _compare(res, want)
    # argmax rows are unique: every planted row decides the same way on both sides
    a = res["accept"].numpy()
    assert ((a >= 0) & (a <= B - 1)).all()
    assert np.array_equal(res["out_len"].numpy(), a + 1)


def test_verify_chained_calls_append():
    b, B, V = 8, 8, 151936
    cap = 2 * B
    out = torch.full((b, cap), -1, dtype=torch.int32)
    ol = torch.zeros(b, dtype=torch.int32)
    seq = torch.full((b,), 50, dtype=torch.int32)
    for it in range(2):
        case = synth.make_verify_case(b, B, V, f"chain{it}", plant=("geometric", 4.0))
        res = _run(case["logits"], case["draft"], out, ol, seq)
        want = O.verify_batch(case["logits"], case["draft"], out, ol, cap, seq)
        assert res["err"] == 0
        _compare(res, want)
        out, ol, seq = res["out_tokens"], res["out_len"], res["seq_lens"]


def test_verify_workspace_reuse_across_batches_and_calls():
    """One workspace serves verify calls of different batch sizes (each request's
    chunk CTAs count themselves in a per-request counter that the last of them
    sets back to zero), with a draft call on the same workspace in between."""
    V = 151936
    cfg = synth.get_config("qwen3_8b_bs32")
    from synth.configs import shrink
    from tests.gpu_common import built
    small = shrink(cfg, L=1, V=2048, batch=4, ctx=("fixed", 40), I=512, d=512, H_t=512).replace(
        name="verify_ws_reuse")
    bm = built(small)
    ws = D.new_workspace(max(bm.model.workspace_size(40, 8, 0), D.verify_workspace_size(40, 8, V)))
    kc, vc = synth.make_kv_cache(small, bm.cap, dtype=bm.model.cache_dtype)
    kc, vc = kc.cuda(), vc.cuda()
    for it, (b, B) in enumerate([(40, 8), (3, 8), (40, 4), (1, 8), (40, 8)]):
        case = synth.make_verify_case(b, B, V, f"reuse{it}", plant=("uniform",), adversarial=True)
        cap = 2 * B
        out0 = torch.full((b, cap), -1, dtype=torch.int32)
        ol0 = torch.zeros(b, dtype=torch.int32)
        seq0 = torch.full((b,), 77, dtype=torch.int32)
        res = _run(case["logits"], case["draft"], out0, ol0, seq0, ws=ws)
        want = O.verify_batch(case["logits"], case["draft"], out0, ol0, cap, seq0)
        assert res["err"] == 0
        _compare(res, want)
        # a draft call between verifies writes its own buffers in the same workspace
        anchors = torch.arange(small.batch, dtype=torch.int32).cuda()
        ctx = torch.full((small.batch,), 40, dtype=torch.int32).cuda()
        out = torch.zeros((small.batch, 8), dtype=torch.int32, device="cuda")
        D.draft_block(bm.model, anchors, ctx, kc, vc, 8, 1, out, ws)
        torch.cuda.synchronize()
        assert D.get_error(ws) == 0


@pytest.mark.parametrize("V", [1024, 1001, 7])
def test_verify_fp32_and_ragged_vocab(V):
    b, B = 3, 4
    case = synth.make_verify_case(b, B, V, "f32", plant=("uniform",), dtype="f32")
    cap = 8
    out0 = torch.full((b, cap), -1, dtype=torch.int32)
    ol0 = torch.zeros(b, dtype=torch.int32)
    seq0 = torch.full((b,), 128, dtype=torch.int32)
    res = _run(case["logits"], case["draft"], out0, ol0, seq0)
    want = O.verify_batch(case["logits"], case["draft"], out0, ol0, cap, seq0)
    assert res["err"] == 0
    _compare(res, want)


def test_verify_exact_ties_and_ulps():
    b, B, V = 2, 4, 4096
    logits = torch.zeros((b, B, V), dtype=torch.bfloat16)
    draft = torch.tensor([[0, 10, 20, 30], [0, 2000, 7, 9]], dtype=torch.int32)
    # request 0: row 0 ties at 10 and 3000 -> 10 (lower); row 1: tie 5 and 20 -> 5 != 20
    logits[0, 0, 10] = 3.0
    logits[0, 0, 3000] = 3.0
    logits[0, 1, 20] = 3.0
    logits[0, 1, 5] = 3.0
    # request 1: row 0 has 2000 one bf16 ulp above 1.0 and 100 at 1.0 -> 2000
    one = torch.tensor(1.0, dtype=torch.bfloat16)
    logits[1, 0, 100] = one
    logits[1, 0, 2000] = (one.view(torch.int16) + 1).view(torch.bfloat16)
    cap = 8
    out0 = torch.full((b, cap), -1, dtype=torch.int32)
    ol0 = torch.zeros(b, dtype=torch.int32)
    seq0 = torch.zeros(b, dtype=torch.int32)
    res = _run(logits, draft, out0, ol0, seq0)
    want = O.verify_batch(logits, draft, out0, ol0, cap, seq0)
    _compare(res, want)
    assert res["accept"].tolist() == [1, 1]
    assert res["out_tokens"][0, :2].tolist() == [10, 5]


def test_verify_errors_write_nothing():
    b, B, V = 4, 8, 151936
    case = synth.make_verify_case(b, B, V, "errs", plant=("uniform",))
    draft = case["draft"].clone()
    draft[1, 3] = V          # token id outside the vocabulary
    draft[2, 5] = -1
    cap = 2
    out0 = torch.full((b, cap), -1, dtype=torch.int32)
    ol0 = torch.tensor([0, 0, 0, 1], dtype=torch.int32)
    seq0 = torch.full((b,), 10, dtype=torch.int32)
    res = _run(case["logits"], draft, out0, ol0, seq0)
    want = O.verify_batch(case["logits"], draft, out0, ol0, cap, seq0)
    assert want["status"][1] == O.VERIFY_TOKEN_RANGE and want["status"][2] == O.VERIFY_TOKEN_RANGE
    exp_bits = D.DEV_TOKEN_RANGE | (D.DEV_OUT_CAP if (want["status"] == O.VERIFY_OUT_CAP).any() else 0)
    assert res["err"] == exp_bits
    _compare(res, want)
    for r in range(b):
        if want["status"][r] != O.VERIFY_OK:
            assert int(res["accept"][r]) == -9 and int(res["next_anchor"][r]) == -9
    # the error word was cleared by the read
    ws = D.new_workspace(D.verify_workspace_size(b, B, V))
    assert D.get_error(ws) == 0
