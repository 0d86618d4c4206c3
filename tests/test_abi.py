"""The C ABI loads, exports every declared symbol and rejects bad arguments on the host.

No call here reaches the GPU: every case fails host-side argument checks first.
"""

import ctypes

import pytest

from block_diffusion_speculative_gemm_b200 import dflash as D


def test_library_exports_every_declared_symbol():
    L = D.lib()
    names = D.header_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    assert D.status_str(D.OK) == "ok"
    assert "invalid" in D.status_str(D.EINVAL)
    assert D.status_str(-99) == "unknown status"


def test_model_create_rejects_null_and_bad_config():
    L = D.lib()
    h = ctypes.c_void_p()
    assert L.dflash_model_create(None, None, ctypes.byref(h)) == D.EINVAL
    cfg = D.Config(dtype=7, H_t=64, n_tap=1, n_layers=1, d=64, n_q=2, n_kv=1, head_dim=64,
                   inter=64, vocab=128, mask_id=127, max_pos=64, eps=1e-6, rope_base=1e6)
    lw = (D.LayerWeights * 1)()
    w = D.Weights(layers=lw)
    assert L.dflash_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == D.EINVAL
    cfg.dtype = D.BF16
    cfg.n_q = 3  # not a multiple of n_kv = 2
    cfg.n_kv = 2
    assert L.dflash_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == D.EINVAL
    cfg.n_q, cfg.n_kv, cfg.head_dim = 2, 1, 96  # head_dim 96 not built
    assert L.dflash_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == D.EUNSUPPORTED
    cfg.head_dim, cfg.d = 64, 4160  # rows wider than the row kernels hold (d <= 4096)
    assert L.dflash_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == D.EINVAL
    cfg.d = 64
    assert h.value is None
    assert L.dflash_model_destroy(None) == D.OK


def test_size_queries_without_model():
    L = D.lib()
    assert L.dflash_workspace_size(None, 4, 8, 100) == 0
    hdr = L.dflash_verify_workspace_size(0, 8, 100)  # the header alone: error word + counters
    assert 256 <= hdr <= (1 << 18) and hdr % 256 == 0
    assert L.dflash_verify_workspace_size(4, 8, 151936) > hdr
    assert L.dflash_verify_workspace_size(-1, 8, 100) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(B=1), D.EINVAL),          # block of one: nothing to verify
    (dict(B=33), D.EINVAL),         # more rows than one warp handles
    (dict(V=0), D.EINVAL),
    (dict(out_cap=0), D.EINVAL),
    (dict(dtype=5), D.EINVAL),
    (dict(logits=None), D.EINVAL),  # null pointers
    (dict(logits=8), D.EINVAL),     # misaligned logits
    (dict(ws=64), D.EINVAL),        # workspace not 256-byte aligned
    (dict(ws_bytes=8), D.EWORKSPACE),
    (dict(batch=0), D.OK),          # nothing to do
])
def test_verify_host_checks(kw, code):
    L = D.lib()
    a = dict(logits=4096, dtype=D.BF16, draft=4096, batch=2, B=4, V=1000, out=4096, out_len=4096,
             out_cap=16, seq=4096, acc=4096, nxt=4096, ws=4096, ws_bytes=1 << 20)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    st = L.dflash_verify(vp(a["logits"]), a["dtype"], vp(a["draft"]), a["batch"], a["B"], a["V"],
                         vp(a["out"]), vp(a["out_len"]), a["out_cap"], vp(a["seq"]), vp(a["acc"]),
                         vp(a["nxt"]), vp(a["ws"]), a["ws_bytes"], None)
    assert st == code


def test_draft_and_inject_reject_null_model_and_bad_block():
    L = D.lib()
    p = ctypes.c_void_p(4096)
    assert L.dflash_draft_block(None, p, p, p, p, 64, 1, 8, 2, p, None, None, p, 1 << 20, None) == D.EINVAL
    assert L.dflash_inject_kv(None, None, p, p, 1, 4, p, p, 64, p, 1 << 20, None) == D.EINVAL
    assert L.dflash_workspace_init(ctypes.c_void_p(4100), 256, None) == D.EINVAL
    assert L.dflash_get_error(None, None, None) == D.EINVAL


def test_sampled_verify_size_query():
    L = D.lib()
    hdr = L.dflash_verify_sampled_workspace_size(0, 8, 100)
    assert hdr == L.dflash_verify_workspace_size(0, 8, 100)  # the shared header alone
    big = L.dflash_verify_sampled_workspace_size(32, 8, 151936)
    assert big > hdr and big % 256 == 0
    assert L.dflash_verify_sampled_workspace_size(-1, 8, 100) == 0
    assert L.dflash_verify_sampled_workspace_size(4, 8, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(B=1), D.EINVAL),
    (dict(B=33), D.EINVAL),
    (dict(V=0), D.EINVAL),
    (dict(out_cap=0), D.EINVAL),
    (dict(dtype=5), D.EINVAL),
    (dict(tau=0.0), D.EINVAL),            # greedy is dflash_verify
    (dict(tau=-1.0), D.EINVAL),
    (dict(tau=float("nan")), D.EINVAL),
    (dict(tau=1e5), D.EINVAL),
    (dict(logits=None), D.EINVAL),
    (dict(dlogits=None), D.EINVAL),
    (dict(dlogits=4104), D.EINVAL),       # misaligned draft logits
    (dict(ws=64), D.EINVAL),
    (dict(batch=20000, B=2), D.EUNSUPPORTED),  # 2 * batch * B rows > 65535
    (dict(ws_bytes=8), D.EWORKSPACE),
    (dict(batch=0), D.OK),
])
def test_sampled_verify_host_checks(kw, code):
    L = D.lib()
    a = dict(logits=4096, dlogits=8192, dtype=D.BF16, draft=4096, batch=2, B=4, V=1000, tau=0.7,
             out=4096, out_len=4096, out_cap=16, seq=4096, acc=4096, nxt=4096, ws=4096,
             ws_bytes=1 << 20)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    st = L.dflash_verify_sampled(vp(a["logits"]), vp(a["dlogits"]), a["dtype"], vp(a["draft"]),
                                 a["batch"], a["B"], a["V"], a["tau"], 1, 0, vp(a["out"]),
                                 vp(a["out_len"]), a["out_cap"], vp(a["seq"]), vp(a["acc"]),
                                 vp(a["nxt"]), vp(a["ws"]), a["ws_bytes"], None)
    assert st == code


def test_sampled_and_paged_calls_reject_null_model_and_bad_arguments():
    L = D.lib()
    p = ctypes.c_void_p(4096)
    # sampled drafting: no model, bad temperature, bad output type
    assert L.dflash_draft_block_sampled(None, p, p, p, p, 64, 1, 8, 2, 1.0, 1, 0, p, None, p,
                                        D.F32, p, 1 << 20, None) == D.EINVAL
    # paged calls: no model
    assert L.dflash_inject_kv_paged(None, None, p, p, 1, 4, p, p, 8, 64, p, 4, p, 1 << 20,
                                    None) == D.EINVAL
    assert L.dflash_draft_block_paged(None, p, p, p, p, 8, 64, p, 4, 1, 8, 2, p, None, None, p,
                                      1 << 20, None) == D.EINVAL


def test_bounds_checked_build_exports_the_same_symbols():
    from block_diffusion_speculative_gemm_b200 import build as Bld

    lib = ctypes.CDLL(Bld.build(checked=True))
    for n in D.header_symbols():
        assert hasattr(lib, n), n
