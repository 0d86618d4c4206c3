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


def test_graphed_cycles_chain_matches_the_oracle():
    """Three replays of one captured cycle whose draft reads its anchors and context
    lengths from the previous verify on the device, each compared with the oracle's
    own cycle, whose anchors and lengths come from the oracle's previous verify.

    Per cycle: the injected K/V rows (1e-2 of max |oracle|); the draft of every
    request under the draft rules (tokens and commit sets, near-ties admitted only
    inside the oracle's bands), drafted over the oracle's own cache (the seeded
    initial contents with the oracle's fp64 injection written over them); verify
    outputs, accept lengths, next anchors and lengths bit-exact, from the GPU's
    admitted draft.  Before each replay, the target logits are planted against the
    oracle's draft of that cycle, so accept lengths span 0..B-1 and the output
    compaction is exercised."""
    import numpy as np

    import oracle as O
    from tests.gpu_common import DraftReport, check_draft_request, rel_err, REL_TOL

    base = synth.get_config("qwen3_8b_bs32")
    cfg = shrink(base, L=2, V=2048, batch=4, ctx=("uniform", 40, 300), I=512, d=512,
                 H_t=512).replace(name="chain_oracle8b")
    B, V, n_cycles = cfg.B, cfg.V, 3
    b = built(cfg, cap=cfg.cache_cap + n_cycles * B + 16)
    dev = torch.device("cuda")
    ctx = synth.make_ctx_lens(cfg)
    anchors0 = synth.make_anchors(cfg)
    cu, st, n = synth.make_inject_layout(cfg, ctx, "steady")
    taps = synth.make_tap_hiddens(cfg, n, label="chain_oracle_taps")
    taps_d = [t.to(dev) for t in taps]
    cu_d, st_d = cu.to(dev), st.to(dev)
    ws = D.new_workspace(max(b.model.workspace_size(cfg.batch, B, n),
                             D.verify_workspace_size(cfg.batch, B, V)))
    kc0, vc0 = synth.make_kv_cache(cfg, b.cap, dtype=b.model.cache_dtype)
    out_cap = n_cycles * B
    s = dict(kc=kc0.to(dev), vc=vc0.to(dev),
             draft=torch.zeros((cfg.batch, B), dtype=torch.int32, device=dev),
             cst=torch.zeros((cfg.batch, B), dtype=torch.int32, device=dev),
             out=torch.full((cfg.batch, out_cap), -1, dtype=torch.int32, device=dev),
             out_len=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
             seq=ctx.clone().to(dev),
             acc=torch.zeros(cfg.batch, dtype=torch.int32, device=dev),
             nxt=anchors0.clone().to(dev))
    logits = torch.zeros((cfg.batch, B, V), dtype=torch.bfloat16, device=dev)

    def cycle():
        D.inject_kv(b.model, taps_d, cu_d, st_d, s["kc"], s["vc"], ws)
        D.draft_block(b.model, s["nxt"], s["seq"], s["kc"], s["vc"], B, cfg.steps, s["draft"],
                      ws, commit_step=s["cst"])
        D.verify(logits, s["draft"], s["out"], s["out_len"], s["seq"], s["acc"], s["nxt"], ws)

    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cycle()
    torch.cuda.synchronize()

    # the oracle's cache: the seeded initial contents, with its own injection over them
    inj = O.inject_kv_requests(taps, cu, st, b.W, cfg)
    caches = []
    for r in range(cfg.batch):
        per = []
        for l in range(cfg.L):
            K = O.as_f64(kc0[l, r]).transpose(1, 0, 2).copy()
            Vv = O.as_f64(vc0[l, r]).transpose(1, 0, 2).copy()
            pos, Ki, Vi = inj[(l, r)]
            K[pos], Vv[pos] = Ki, Vi
            per.append((K, Vv))
        caches.append(per)
    o_anchor = anchors0.numpy().astype(np.int64)
    o_seq = ctx.numpy().astype(np.int64)
    o_out = np.full((cfg.batch, out_cap), -1, dtype=np.int64)
    o_len = np.zeros(cfg.batch, dtype=np.int64)
    rep = DraftReport()
    accepts = []
    for c in range(n_cycles):
        # plant this cycle's target logits against the oracle's draft
        o_draft = np.stack([O.draft_block(int(o_anchor[r]), int(o_seq[r]),
                                          [(K[:o_seq[r]], Vv[:o_seq[r]]) for K, Vv in caches[r]],
                                          b.W, cfg)[0] for r in range(cfg.batch)])
        case = synth.make_verify_case(cfg.batch, B, V, f"chain_oracle{c}", plant=("uniform",),
                                      draft=torch.as_tensor(o_draft, dtype=torch.int32))
        logits.copy_(case["logits"].to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert D.get_error(ws) == 0
        # injection (the same rows every cycle)
        for l in range(cfg.L):
            for r in range(cfg.batch):
                pos, Ki, Vi = inj[(l, r)]
                gk = s["kc"][l, r, :, torch.as_tensor(pos)].float().cpu().numpy().transpose(1, 0, 2)
                gv = s["vc"][l, r, :, torch.as_tensor(pos)].float().cpu().numpy().transpose(1, 0, 2)
                assert rel_err(gk, Ki) <= REL_TOL and rel_err(gv, Vi) <= REL_TOL, (c, l, r)
        draft = s["draft"].cpu()
        cst = s["cst"].cpu()
        for r in range(cfg.batch):
            T = int(o_seq[r])
            check_draft_request(b, r, int(o_anchor[r]), T,
                                [(K[:T], Vv[:T]) for K, Vv in caches[r]], draft[r], cst[r],
                                None, cfg.steps, rep)
        vr = O.verify_batch(case["logits"], draft, o_out, o_len, out_cap, o_seq)
        assert (vr["status"] == 0).all()
        assert np.array_equal(s["out"].cpu().numpy(), vr["out_tokens"]), c
        assert np.array_equal(s["out_len"].cpu().numpy(), vr["out_len"]), c
        assert np.array_equal(s["seq"].cpu().numpy(), vr["seq_lens"]), c
        assert np.array_equal(s["acc"].cpu().numpy(), vr["accept"]), c
        assert np.array_equal(s["nxt"].cpu().numpy(), vr["next_anchor"]), c
        accepts += [int(a) for a in vr["accept"]]
        o_anchor, o_seq = vr["next_anchor"], vr["seq_lens"]
        o_out, o_len = vr["out_tokens"], vr["out_len"]
    assert max(accepts) > 0  # the planted prefixes were accepted somewhere
    rep.save("graph_chain_vs_oracle", config=cfg.name, cycles=n_cycles, accepts=accepts)
    print(rep, accepts)
