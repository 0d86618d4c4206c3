"""fp16 range guard of the bf16 model type (which multiplies fp16 x fp16 on the
tensor cores and stores fp16 activations and K/V).

* A bf16 weight past fp16's finite range (a planted 7e4) makes model creation
  fail with DFLASH_EUNSUPPORTED instead of turning into an infinity.
* An activation that overflows fp16 (a planted norm gain of 3e4 makes RMSNorm
  outputs of ~1e5) sets DFLASH_DEV_RANGE in the device error word, in
  injection (the context-feature norm) and in drafting (the layer norms).
"""

import pytest
import torch

import synth
from synth.configs import shrink
from synth.device import to_device
from tests.gpu_common import max_pos_for
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def _cfg():
    base = synth.get_config("qwen3_8b_bs32")
    return shrink(base, L=1, V=2048, batch=2, ctx=("fixed", 64), I=512, d=512,
                  H_t=512).replace(name="range8b")


def test_out_of_range_weight_is_refused():
    cfg = _cfg()
    w = synth.make_weights(cfg)
    w["layers"][0]["Wd"][3, 5] = 7e4
    with pytest.raises(D.DFlashError) as e:
        D.Model(cfg, to_device(w), max_pos_for(cfg))
    assert e.value.status == D.EUNSUPPORTED
    # the same weights without the planted value load
    w["layers"][0]["Wd"][3, 5] = 0.01
    D.Model(cfg, to_device(w), max_pos_for(cfg)).close()


def test_activation_overflow_sets_the_range_bit():
    cfg = _cfg()
    w = synth.make_weights(cfg)
    w["g_ctx"].fill_(3e4)
    w["layers"][0]["g_post"].fill_(3e4)
    model = D.Model(cfg, to_device(w), max_pos_for(cfg))
    try:
        cap = cfg.cache_cap
        ctx = synth.make_ctx_lens(cfg)
        cu, st, n = synth.make_inject_layout(cfg, ctx, "prefill")
        taps = [t.cuda() for t in synth.make_tap_hiddens(cfg, n)]
        kc = torch.zeros((cfg.L, cfg.batch, cfg.nkv, cap, cfg.hd), dtype=model.cache_dtype,
                         device="cuda")
        vc = torch.zeros_like(kc)
        ws = model.workspace(cfg.batch, cfg.B, n)
        D.inject_kv(model, taps, cu.cuda(), st.cuda(), kc, vc, ws)
        assert D.get_error(ws) & D.DEV_RANGE
        out = torch.zeros((cfg.batch, cfg.B), dtype=torch.int32, device="cuda")
        D.draft_block(model, synth.make_anchors(cfg).cuda(), ctx.cuda(), kc, vc, cfg.B,
                      cfg.steps, out, ws)
        assert D.get_error(ws) & D.DEV_RANGE
    finally:
        model.close()
