"""dflash_verify_noalloc: greedy verify for callers that cannot allocate device memory.

A serving engine that reserves all of its device memory in its own pool at
start-up (and allows no allocation afterwards), or a plugin living inside
another framework's allocator, cannot hand the library a workspace.  This entry
point keeps its scratch in a fixed array inside the library.  Here it is called
through the C ABI (ctypes) and must match dflash_verify exactly, on two calls in
a row that append to the same output buffers.  The file sorts last so that a run
stopping at its first failure has already run every other test.
"""

import ctypes

import pytest
import torch

import synth
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def _buffers(b, B, cap, seq0):
    return dict(out=torch.full((b, cap), -1, dtype=torch.int32, device="cuda"),
                out_len=torch.zeros(b, dtype=torch.int32, device="cuda"),
                seq=seq0.clone().cuda(),
                acc=torch.full((b,), -9, dtype=torch.int32, device="cuda"),
                nxt=torch.full((b,), -9, dtype=torch.int32, device="cuda"))


def _noalloc_abi(logits, draft, o, err):
    """Direct C-ABI call (no binding helper), as a non-Python caller would make it."""
    L = D.lib()
    b, B, V = logits.shape
    dt = D.BF16 if logits.dtype == torch.bfloat16 else D.F32
    st = L.dflash_verify_noalloc(
        ctypes.c_void_p(logits.data_ptr()), dt, ctypes.c_void_p(draft.data_ptr()), b, B, V,
        ctypes.c_void_p(o["out"].data_ptr()), ctypes.c_void_p(o["out_len"].data_ptr()),
        o["out"].shape[1], ctypes.c_void_p(o["seq"].data_ptr()),
        ctypes.c_void_p(o["acc"].data_ptr()), ctypes.c_void_p(o["nxt"].data_ptr()),
        ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == D.OK, D.status_str(st)


@pytest.mark.parametrize("b,B,V,dtype", [(32, 8, 151936, "bf16"), (3, 4, 1001, "f32"),
                                         (128, 16, 151936, "bf16")])
def test_noalloc_verify_matches_workspace_verify_twice(b, B, V, dtype):
    cap = 2 * B + 1
    seq0 = torch.randint(100, 5000, (b,), dtype=torch.int32)
    ref = _buffers(b, B, cap, seq0)
    got = _buffers(b, B, cap, seq0)
    ws = D.new_workspace(D.verify_workspace_size(b, B, V))
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        case = synth.make_verify_case(b, B, V, f"noalloc{call}", plant=("geometric", 4.0),
                                      dtype=dtype, adversarial=(call == 1))
        logits, draft = case["logits"].cuda(), case["draft"].cuda()
        D.verify(logits, draft, ref["out"], ref["out_len"], ref["seq"], ref["acc"], ref["nxt"], ws)
        _noalloc_abi(logits, draft, got, err)
        torch.cuda.synchronize()
        assert D.get_error(ws) == 0
        assert int(err.item()) == 0
        for k in ref:
            assert torch.equal(ref[k], got[k]), (call, k)


def test_noalloc_reports_device_errors_and_rejects_oversize():
    b, B, V = 4, 8, 151936
    case = synth.make_verify_case(b, B, V, "noalloc_err")
    draft = case["draft"].clone()
    draft[2, 3] = V  # outside the vocabulary: that request writes nothing
    o = _buffers(b, B, 2 * B, torch.full((b,), 7, dtype=torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    D.verify_noalloc(case["logits"].cuda(), draft.cuda(), o["out"], o["out_len"], o["seq"],
                     o["acc"], o["nxt"], err)
    torch.cuda.synchronize()
    assert int(err.item()) == D.DEV_TOKEN_RANGE
    assert int(o["acc"][2]) == -9 and int(o["out_len"][2]) == 0
    # the next call starts from a clear error word
    D.verify_noalloc(case["logits"].cuda(), case["draft"].cuda(), o["out"], o["out_len"], o["seq"],
                     o["acc"], o["nxt"], err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # a request beyond the fixed scratch is refused before anything runs
    L = D.lib()
    p = ctypes.c_void_p(case["logits"].cuda().data_ptr())
    st = L.dflash_verify_noalloc(p, D.BF16, p, 2100, 16, V, p, p, 8, p, p, p, None, None)
    assert st == D.ESCRATCH  # 33600 rows > 32768


def test_noalloc_allocates_nothing():
    """After a first call (which may load the module that holds the fixed array),
    further calls at the largest parametrised shape leave the device's free memory
    unchanged: no call allocates device memory."""
    b, B, V = 128, 16, 151936
    n_calls = 5
    case = synth.make_verify_case(b, B, V, "noalloc_mem", plant=("geometric", 4.0))
    logits, draft = case["logits"].cuda(), case["draft"].cuda()
    o = _buffers(b, B, (n_calls + 1) * B, torch.full((b,), 11, dtype=torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _noalloc_abi(logits, draft, o, err)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(n_calls):
        _noalloc_abi(logits, draft, o, err)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(err.item()) == 0
    assert (o["out_len"].cpu() > n_calls).all()
