"""The three hot calls, captured in a CUDA graph and replayed, give the same
results as launching them directly: no call allocates, synchronises or reads
device memory on the host, and the dependent-launch chain survives capture."""

import pytest
import torch

import synth
from synth.configs import shrink
from tests.gpu_common import built
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu


def test_cycle_graph_replay_matches_eager():
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=4096, batch=6, ctx=("uniform", 40, 600), I=1024, d=1024,
                 H_t=512).replace(name="graph8b")
    b = built(cfg)
    dev = torch.device("cuda")
    B, V = cfg.B, cfg.V
    ctx = synth.make_ctx_lens(cfg)
    anchors = synth.make_anchors(cfg)
    cu, st, n = synth.make_inject_layout(cfg, ctx, "steady")
    taps = [t.to(dev) for t in synth.make_tap_hiddens(cfg, n, label="graph_taps")]
    case = synth.make_verify_case(cfg.batch, B, V, "graph", plant=("uniform",))
    logits = case["logits"].to(dev)
    ws = D.new_workspace(max(b.model.workspace_size(cfg.batch, B, n),
                             D.verify_workspace_size(cfg.batch, B, V)))
    cap = 4 * B

    def fresh():
        kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
        return dict(kc=kc.to(dev), vc=vc.to(dev),
                    draft=torch.zeros((cfg.batch, B), dtype=torch.int32, device=dev),
                    out=torch.full((cfg.batch, cap), -1, dtype=torch.int32, device=dev),
                    out_len=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
                    seq=ctx.clone().to(dev),
                    acc=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
                    nxt=torch.zeros(cfg.batch, dtype=torch.int32, device=dev))

    def cycle(s):
        D.inject_kv(b.model, taps, cu.to(dev), st.to(dev), s["kc"], s["vc"], ws)
        D.draft_block(b.model, anchors.to(dev), ctx.to(dev), s["kc"], s["vc"], B, cfg.steps,
                      s["draft"], ws)
        D.verify(logits, s["draft"], s["out"], s["out_len"], s["seq"], s["acc"], s["nxt"], ws)

    eager = fresh()
    cycle(eager)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0

    graphed = fresh()
    cu_d, st_d, an_d, ctx_d = cu.to(dev), st.to(dev), anchors.to(dev), ctx.to(dev)

    def cycle_dev(s):
        D.inject_kv(b.model, taps, cu_d, st_d, s["kc"], s["vc"], ws)
        D.draft_block(b.model, an_d, ctx_d, s["kc"], s["vc"], B, cfg.steps, s["draft"], ws)
        D.verify(logits, s["draft"], s["out"], s["out_len"], s["seq"], s["acc"], s["nxt"], ws)

    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cycle_dev(graphed)
    g.replay()
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    for k in ("kc", "vc", "draft", "out", "out_len", "seq", "acc", "nxt"):
        assert torch.equal(eager[k], graphed[k]), k


def test_graphed_cycles_chain_anchors_and_lengths_on_device():
    """A captured cycle whose draft takes its anchors from the previous verify's
    next_anchor and its context lengths from the updated seq_lens: replaying it
    three times gives what three directly launched cycles give."""
    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=1, V=2048, batch=4, ctx=("uniform", 40, 300), I=512, d=512,
                 H_t=512).replace(name="chain8b")
    B, V, n_cycles = cfg.B, cfg.V, 3
    # every cycle lengthens each context by up to B accepted tokens
    b = built(cfg, cap=cfg.cache_cap + n_cycles * B + 16)
    dev = torch.device("cuda")
    ctx = synth.make_ctx_lens(cfg)
    cu, st, n = synth.make_inject_layout(cfg, ctx, "steady")
    taps = [t.to(dev) for t in synth.make_tap_hiddens(cfg, n, label="chain_taps")]
    case = synth.make_verify_case(cfg.batch, B, V, "chain", plant=("uniform",))
    logits = case["logits"].to(dev)
    ws = D.new_workspace(max(b.model.workspace_size(cfg.batch, B, n),
                             D.verify_workspace_size(cfg.batch, B, V)))
    cu_d, st_d = cu.to(dev), st.to(dev)

    def fresh():
        kc, vc = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
        return dict(kc=kc.to(dev), vc=vc.to(dev),
                    draft=torch.zeros((cfg.batch, B), dtype=torch.int32, device=dev),
                    out=torch.full((cfg.batch, n_cycles * B), -1, dtype=torch.int32, device=dev),
                    out_len=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
                    seq=ctx.clone().to(dev),
                    acc=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
                    nxt=synth.make_anchors(cfg).to(dev))

    def cycle(s):
        D.inject_kv(b.model, taps, cu_d, st_d, s["kc"], s["vc"], ws)
        # anchors and context lengths come from the previous verify, on the device
        D.draft_block(b.model, s["nxt"], s["seq"], s["kc"], s["vc"], B, cfg.steps, s["draft"], ws)
        D.verify(logits, s["draft"], s["out"], s["out_len"], s["seq"], s["acc"], s["nxt"], ws)

    eager = fresh()
    for _ in range(n_cycles):
        cycle(eager)
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    assert (eager["out_len"].cpu() >= n_cycles).all()

    graphed = fresh()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cycle(graphed)
    for _ in range(n_cycles):
        g.replay()
    torch.cuda.synchronize()
    assert D.get_error(ws) == 0
    for k in ("kc", "vc", "draft", "out", "out_len", "seq", "acc", "nxt"):
        assert torch.equal(eager[k], graphed[k]), k
