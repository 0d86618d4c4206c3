"""Failure detection without a fault: a bounded wait that nothing completes gives
up after its limit, reports DFLASH_DEV_TIMEOUT through the workspace error word,
and leaves the context usable."""

import time

import pytest
import torch

import synth
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = D.new_workspace(256)
    t0 = time.perf_counter()
    assert D.lib().dflash_debug_wait_timeout(D._ptr(ws), D._stream(None)) == 0
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert D.get_error(ws) == D.DEV_TIMEOUT
    assert 0.9 < waited < 30.0
    assert D.get_error(ws) == 0  # read and cleared
    # the context still runs the hot path
    b, B, V = 2, 4, 1024
    case = synth.make_verify_case(b, B, V, "after_timeout", plant=("uniform",))
    out = torch.full((b, 2 * B), -1, dtype=torch.int32, device="cuda")
    ol = torch.zeros(b, dtype=torch.int32, device="cuda")
    seq = torch.zeros(b, dtype=torch.int32, device="cuda")
    acc = torch.zeros(b, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(b, dtype=torch.int32, device="cuda")
    vws = D.new_workspace(D.verify_workspace_size(b, B, V))
    D.verify(case["logits"].cuda(), case["draft"].cuda(), out, ol, seq, acc, nxt, vws)
    torch.cuda.synchronize()
    assert D.get_error(vws) == 0
    assert (ol.cpu() >= 1).all()
