"""Benchmark of the DFlash draft hot path on B200.

One step = one whole cycle of the hot path over the Qwen3-8B-shaped workload
with 32 requests (contexts uniform in [512, 4096], block 8, two denoising
steps): KV injection of the rows accepted in the previous cycle, the masked
block draft (both denoising steps) and greedy verify of the block against
given target logits.  Metric: block tokens per second of that cycle
(32 * 8 tokens drafted and verified per step); the JSON line also carries the
draft-only and verify-only rates, the per-kernel-class device times and the
roofline of the dominant kernel class.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dflash|reference]

Multi-GPU: one process per GPU (torchrun), every rank runs its own 32
requests (requests are independent: no data-path collective), max time over
ranks, value = all ranks' tokens / that time.  `--impl reference` times the
fp64 CPU oracle on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth.device import to_device  # noqa: E402

WORKLOAD = "qwen3_8b_bs32"
METRIC = "draft-block tokens/s + verify rows/s at 8B-shape bs32, % of HBM/TC roofline"
UNIT = "block tok/s"


# ------------------------------------------------------------------ helpers

def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's value (a device time): the job is as slow as its
    slowest replica."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(per_rank_units: int, world: int, ms_per_step: float) -> float:
    """Whole-job units per second: every rank processes its own units each step."""
    return per_rank_units * world / (ms_per_step / 1e3)


def load_peaks():
    """HBM copy bandwidth and bf16 tensor peaks: the measured figures when
    MEASURED_PEAKS.json is present, else the pool's earlier measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def tensor_peak(peaks, clocks):
    """The bf16 tensor peak that matches the clock a timed region ran at: the burst
    figure while the sampled median SM clock stays within 5% of its maximum (a short
    region, before the power cap lowers the clock), else the sustained figure
    measured under the power cap.  Returns (TFLOP/s, "burst" | "sustained")."""
    sm, mx = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    sus = peaks.get("bf16_tflops_sustained")
    if sus and not (sm and mx and sm >= 0.95 * mx):
        return float(sus), "sustained"
    return float(peaks["bf16_tflops"]), "burst"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 50):
        self.idx = device_index
        self.period = period_ms
        self.proc = None
        self.samples = []  # (arrival time, csv line)
        self.lines = []
        self.thread = None
        self.t0 = self.t1 = 0.0

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.samples.append((time.monotonic(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 f"-lms={self.period}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # the timed region starts once the sampler is producing samples
            deadline = time.monotonic() + 3.0
            while not self.samples and time.monotonic() < deadline:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        self.t1 = time.monotonic()
        if self.proc is not None:
            time.sleep(self.period / 1000.0 + 0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            if self.thread is not None:
                self.thread.join(timeout=5)
            # samples taken while the timed region ran
            self.lines = [l for t, l in self.samples
                          if self.t0 <= t <= self.t1 + self.period / 1000.0]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gemm_bytes(N, K, M, out_bytes_per_row):
    """Algorithmic bytes of one weight-streaming GEMM: weights + inputs + outputs."""
    return N * K * 2 + M * K * 2 + M * out_bytes_per_row


def step_algorithmic(cfg, n_inject, ctx_lens, peaks, tc_tflops=None):
    """Algorithmic bytes / flops of one cycle per kernel class, and each class's
    roofline time `roof_s`: every GEMM takes the longer of its flops at the bf16
    tensor peak `tc_tflops` (default: the sustained figure) and its bytes at the HBM
    peak; attention and verify are bytes at the HBM peak."""
    b, B, L, d = cfg.batch, cfg.B, cfg.L, cfg.d
    M = b * B
    q = cfg.nq * cfg.hd
    kv = cfg.nkv * cfg.hd
    qkv = q + 2 * kv
    hbm = peaks["hbm_gbs"] * 1e9
    if tc_tflops is None:
        tc_tflops = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    tc = tc_tflops * 1e12
    out = {k: {"bytes": 0, "flops": 0, "roof_s": 0.0, "roof_tensor_s": 0.0}
           for k in ("gemm", "lm_head", "attention", "verify")}

    def gemm(cls, N, K, rows, out_bytes_per_row, times=1):
        by = gemm_bytes(N, K, rows, out_bytes_per_row)
        fl = 2 * N * K * rows
        c = out[cls]
        c["bytes"] += times * by
        c["flops"] += times * fl
        c["roof_s"] += times * max(fl / tc, by / hbm)
        c["roof_tensor_s"] += times * (fl / tc if fl / tc >= by / hbm else 0.0)

    # injection: fc over the concatenated taps, then the layer-batched K/V projection
    for N, K in ((d, cfg.n_tap * cfg.H_t), (L * 2 * kv, d)):
        gemm("gemm", N, K, n_inject, N * 2)
    rem = B - 1
    T = int(ctx_lens.sum())
    for t in range(cfg.steps):
        k = -(-rem // (cfg.steps - t))
        for N, K in ((qkv, d), (d, q), (2 * cfg.I, d), (d, cfg.I)):
            gemm("gemm", N, K, M, N * 2, times=L)
        n_vt = -(-cfg.V // 128)
        gemm("lm_head", cfg.V, d, b * rem, n_vt * 16)
        # attention: context K and V of every layer, plus the block's q/k/v/o rows
        out["attention"]["bytes"] += L * (T * kv * 2 * 2 + M * (2 * q + 2 * kv) * 2)
        rem -= k
    out["verify"]["bytes"] = M * cfg.V * 2 + M * 4 * 2
    for k in ("attention", "verify"):
        out[k]["roof_s"] = out[k]["bytes"] / hbm
    return out


# ------------------------------------------------------------------ GPU arm

def run_dflash(args, rank, world, local_rank):
    from block_diffusion_speculative_gemm_b200 import dflash as D

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.attn_schedule:
        D.debug_attn_schedule(args.attn_schedule)
    cfg = synth.get_config(WORKLOAD)
    if args.layers:
        # profiling variant: the same per-layer shapes with fewer layers (smaller footprint)
        cfg = cfg.replace(L=args.layers, name=f"{WORKLOAD}_L{args.layers}")
    b, B, V = cfg.batch, cfg.B, cfg.V
    cap = cfg.cache_cap
    w = synth.make_weights(cfg)
    model = D.Model(cfg, to_device(w, dev), cap + 2 * B + 16)
    ctx = synth.make_ctx_lens(cfg)
    anchors = synth.make_anchors(cfg)
    kc = torch.zeros((cfg.L, b, cfg.nkv, cap, cfg.hd), dtype=model.cache_dtype, device=dev)
    vc = torch.zeros_like(kc)

    # prefix: inject every context position once (tapped hiddens drawn on the device)
    cu_p, st_p, n_p = synth.make_inject_layout(cfg, ctx, "prefill")
    cu_s, st_s, n_s = synth.make_inject_layout(cfg, ctx, "steady")
    ws = model.workspace(b, B, max(n_s, 16384))
    gen = torch.Generator(device=dev).manual_seed(synth.sub_seed(0x5EED, WORKLOAD, "prefix"))
    cu_p_d = cu_p.to(dev)
    taps_p = [(torch.randn((n_p, cfg.H_t), generator=gen, device=dev) * cfg.h_std).to(torch.bfloat16)
              for _ in range(cfg.n_tap)]
    st_p_d = st_p.to(dev)
    D.inject_kv(model, taps_p, cu_p_d, st_p_d, kc, vc, ws)
    torch.cuda.synchronize()
    # the prefill injection once more, timed: it rewrites the same cache rows, and at
    # tens of thousands of rows its GEMMs are the tensor-bound part of the path
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    D.inject_kv(model, taps_p, cu_p_d, st_p_d, kc, vc, ws)
    p1.record()
    torch.cuda.synchronize()
    prefill_ms = p0.elapsed_time(p1)
    del taps_p
    assert D.get_error(ws) == 0

    taps_s = [t.to(dev) for t in synth.make_tap_hiddens(cfg, n_s, label="taps_steady")]
    cu_s_d, st_s_d = cu_s.to(dev), st_s.to(dev)
    anchors_d, ctx_d = anchors.to(dev), ctx.to(dev)
    draft = torch.zeros((b, B), dtype=torch.int32, device=dev)
    D.draft_block(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, draft, ws)
    torch.cuda.synchronize()
    # target logits whose greedy argmax agrees with the drafted block on a planted prefix
    case = synth.make_verify_case(b, B, V, "bench", plant=cfg.plant, draft=draft.cpu())
    logits = case["logits"].to(dev)
    # every verify call appends up to B tokens per request: warm-up, timed and
    # per-class timing steps
    steps_total = args.warmup + args.steps + min(args.steps, 20) + 4
    out_cap = steps_total * B
    out_tok = torch.zeros((b, out_cap), dtype=torch.int32, device=dev)
    out_len = torch.zeros(b, dtype=torch.int32, device=dev)
    seq = ctx.clone().to(dev)
    acc = torch.zeros(b, dtype=torch.int32, device=dev)
    nxt = torch.zeros(b, dtype=torch.int32, device=dev)

    def step():
        D.inject_kv(model, taps_s, cu_s_d, st_s_d, kc, vc, ws)
        D.draft_block(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, draft, ws)
        D.verify(logits, draft, out_tok, out_len, seq, acc, nxt, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    # per-class device times from separate steps: the events recorded around each
    # class serialise the kernels they bracket, so they stay out of the timed region
    n_cls = min(args.steps, 20)
    D.timing_read()  # discard
    D.timing_enable(True)
    for _ in range(n_cls):
        step()
    torch.cuda.synchronize()
    D.timing_enable(False)
    per_class = D.timing_read()
    # dflash_draft_block alone (all denoising steps), back to back
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_draft = args.steps
    for _ in range(3):
        D.draft_block(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, draft, ws)
    torch.cuda.synchronize()
    # sampled like the timed region: the draft-only loop runs after seconds of load,
    # where the power cap may have lowered the SM clock
    with ClockSampler(local_rank) as dclk:
        d0.record(stream)
        for _ in range(n_draft):
            D.draft_block(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, draft, ws)
        d1.record(stream)
        torch.cuda.synchronize()
    draft_ms = d0.elapsed_time(d1) / n_draft
    # sampled drafting (temperature 1) over the same caches: the same forwards, the
    # committing-step logits rows written for sampled verify, and a Gumbel-max draw
    # over the vocabulary of every masked row in place of the LM-head argmax
    q_rows = torch.empty((b, B, V), dtype=torch.bfloat16, device=dev)
    draft_s = torch.zeros_like(draft)
    for k in range(3):
        D.draft_block_sampled(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, 1.0, 0x5EED, k,
                              draft_s, q_rows, ws)
    torch.cuda.synchronize()
    d0.record(stream)
    for k in range(n_draft):
        D.draft_block_sampled(model, anchors_d, ctx_d, kc, vc, B, cfg.steps, 1.0, 0x5EED, 3 + k,
                              draft_s, q_rows, ws)
    d1.record(stream)
    torch.cuda.synchronize()
    sampled_ms = d0.elapsed_time(d1) / n_draft
    del q_rows
    err = D.get_error(ws)
    if err:
        raise RuntimeError(f"device error word {err}")
    ms_step = max_over_ranks(ms, world, dev) / args.steps
    value = job_throughput(b * B, world, ms_step)

    # ---- per-class device times (this rank) and the roofline of the dominant class
    peaks = load_peaks()
    clocks = clk.summary()
    tc_peak, tc_kind = tensor_peak(peaks, clocks)
    alg = step_algorithmic(cfg, n_s, ctx, peaks, tc_peak)
    classes = {}
    for name, key in (("gemm", "gemm"), ("attention", "attention"), ("lm_head", "lm_head"),
                      ("verify", "verify"), ("row", "row")):
        c = per_class.get(key, {"ms": 0.0, "launches": 0})
        classes[name] = {"ms_per_step": c["ms"] / n_cls,
                         "launches_per_step": c["launches"] / n_cls}
    for name in ("gemm", "attention", "lm_head", "verify"):
        t = classes[name]["ms_per_step"] / 1e3
        if t > 0:
            c = classes[name]
            c["algorithmic_GBps"] = alg[name]["bytes"] / t / 1e9
            c["frac_hbm"] = c["algorithmic_GBps"] / peaks["hbm_gbs"]
            if alg[name]["flops"]:
                c["TFLOPs"] = alg[name]["flops"] / t / 1e12
                c["frac_tensor"] = c["TFLOPs"] / tc_peak
            c["frac_roofline"] = alg[name]["roof_s"] / t
    dom = max(("gemm", "attention", "lm_head", "verify"), key=lambda n: classes[n]["ms_per_step"])
    # kernels launched inside the timed region: every step launches the same list
    launches = sum(int(c["launches"]) for c in per_class.values()) * args.steps // n_cls
    n_dom = per_class[dom]["launches"] / n_cls
    traffic = load_traffic(dom)
    common = {"kernel": dom, "peak_source": peaks["source"],
              "algorithmic_bytes_per_launch": alg[dom]["bytes"] / max(n_dom, 1),
              "algorithmic_flops_per_launch": alg[dom]["flops"] / max(n_dom, 1),
              "avg_launch_ms": classes[dom]["ms_per_step"] / max(n_dom, 1), "traffic": traffic}
    if alg[dom]["roof_tensor_s"] * 2 > alg[dom]["roof_s"]:
        # mostly compute-bound: against the tensor peak of the clock the step ran at
        achieved = classes[dom]["TFLOPs"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tc_peak,
                "peak_kind": f"bf16 {tc_kind}", "unit": "TFLOP/s",
                "frac": round(achieved / tc_peak, 4), **common}
    else:
        achieved = classes[dom]["algorithmic_GBps"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), **common}
    # whole-cycle roofline: the sum of the classes' roofline times
    roof_ms = sum(alg[n]["roof_s"] for n in ("gemm", "attention", "lm_head", "verify")) * 1e3
    class_sum_ms = sum(classes[n]["ms_per_step"] for n in classes)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and inputs)",
        "config": {"workload": cfg.name, "model": f"Qwen3-8B-shaped DFlash draft ({cfg.L} layers)",
                   "global_batch": b * world, "block": B, "denoise_steps": cfg.steps,
                   "ctx": "uniform[512,4096]", "inject_rows": n_s, "parallelism": f"dp{world}",
                   "attention": ["split-KV grid (chunk planned per forward), mma.sync",
                                 "persistent, mma.sync",
                                 "split-KV grid (chunk planned per forward), tcgen05"][
                                     args.attn_schedule],
                   "l2": "no flush: every step streams ~7.4 GB of weights and K/V (> 126 MB L2)"},
        "roofline": roof,
        "tensor_peak": {"TFLOPs": tc_peak, "kind": tc_kind,
                        "rule": "burst while the median SM clock is within 5% of max, else "
                                "sustained"},
        "cycle_roofline_ms": round(roof_ms, 4),
        "cycle_frac_of_roofline": round(roof_ms / ms_step, 4),
        "classes": classes,
        # events around each class serialise its launches with their neighbours, so
        # the class times sum to more than the overlapped step: every class fraction
        # is a lower bound
        "class_sum_ms": round(class_sum_ms, 4),
        "class_times": "event-bracketed per class (serialised): fractions are lower bounds",
        "gpu_launches": launches,
        "verify_rows_s": round(b * B / (classes["verify"]["ms_per_step"] / 1e3), 1)
        if classes["verify"]["ms_per_step"] > 0 else None,
        # dflash_draft_block alone: block positions and drafted (masked) positions per s
        "draft_block": {"ms": round(draft_ms, 4),
                        "block_tok_s": round(b * world * B / (draft_ms / 1e3), 1),
                        "drafted_tok_s": round(b * world * (B - 1) / (draft_ms / 1e3), 1),
                        "clocks": dclk.summary()},
        # dflash_draft_block_sampled at temperature 1, same loop
        "draft_block_sampled": {"ms": round(sampled_ms, 4),
                                "block_tok_s": round(b * world * B / (sampled_ms / 1e3), 1),
                                "over_greedy": round(sampled_ms / draft_ms, 4)},
        "prefill_inject": prefill_report(cfg, n_p, prefill_ms, peaks),
        "clocks": clocks,
    }
    if rank == 0 and not args.no_e2e:
        res["e2e"] = run_e2e(args, D, model, cfg, taps_s, cu_s, st_s, anchors, ctx, case, kc, vc, ws,
                             dev, world)
    elif world > 1 and not args.no_e2e:
        run_e2e(args, D, model, cfg, taps_s, cu_s, st_s, anchors, ctx, case, kc, vc, ws, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, cfg, ctx, anchors, cu_s, st_s, n_s, case)
    model.close()
    return res


def run_e2e(args, D, model, cfg, taps_s, cu_s, st_s, anchors, ctx, case, kc, vc, ws, dev, world):
    """Same cycle through the public API with host inputs/outputs: every step copies its
    inputs from pinned host memory and reads its results back."""
    b, B = cfg.batch, cfg.B
    h_taps = [t.cpu().pin_memory() for t in taps_s]
    h_small = {k: v.pin_memory() for k, v in dict(cu=cu_s, st=st_s, anchor=anchors, ctx=ctx).items()}
    h_logits = case["logits"].pin_memory()
    d_taps = [torch.empty_like(t) for t in taps_s]
    d_small = {k: torch.empty_like(v, device=dev) for k, v in h_small.items()}
    d_logits = torch.empty_like(h_logits, device=dev)
    draft = torch.zeros((b, B), dtype=torch.int32, device=dev)
    steps = max(3, args.steps // 4)
    out_cap = (steps + 8) * B
    out_tok = torch.zeros((b, out_cap), dtype=torch.int32, device=dev)
    out_len = torch.zeros(b, dtype=torch.int32, device=dev)
    seq = torch.zeros(b, dtype=torch.int32, device=dev)
    acc = torch.zeros(b, dtype=torch.int32, device=dev)
    nxt = torch.zeros(b, dtype=torch.int32, device=dev)
    h_res = {k: torch.empty(v.shape, dtype=torch.int32).pin_memory() for k, v in
             dict(draft=draft, acc=acc, nxt=nxt, out_len=out_len).items()}
    h2d = sum(t.numel() * t.element_size() for t in h_taps) + sum(
        v.numel() * 4 for v in h_small.values()) + h_logits.numel() * 2
    d2h = sum(v.numel() * 4 for v in h_res.values())

    # The target logits are needed only by verify: they cross PCIe on a side stream
    # while injection and drafting run.  Host-to-device copies share one copy
    # engine, so the inputs that injection needs first go before them; the logits
    # copy is ordered after those on the main stream, inside the timed region.
    copy_stream = torch.cuda.Stream(device=dev)
    ev_start, ev_logits = torch.cuda.Event(), torch.cuda.Event()

    def body():
        main = torch.cuda.current_stream()
        for h, d in zip(h_taps, d_taps):
            d.copy_(h, non_blocking=True)
        for k in h_small:
            d_small[k].copy_(h_small[k], non_blocking=True)
        ev_start.record(main)
        copy_stream.wait_event(ev_start)
        with torch.cuda.stream(copy_stream):
            d_logits.copy_(h_logits, non_blocking=True)
            ev_logits.record(copy_stream)
        seq.copy_(d_small["ctx"])
        D.inject_kv(model, d_taps, d_small["cu"], d_small["st"], kc, vc, ws)
        D.draft_block(model, d_small["anchor"], d_small["ctx"], kc, vc, B, cfg.steps, draft, ws)
        main.wait_event(ev_logits)
        D.verify(d_logits, draft, out_tok, out_len, seq, acc, nxt, ws)
        for k, d in (("draft", draft), ("acc", acc), ("nxt", nxt), ("out_len", out_len)):
            h_res[k].copy_(d, non_blocking=True)

    # One step's API calls (copies in, inject, draft, verify, read-back) are captured
    # once into a CUDA graph and replayed every step, as a serving loop would; each
    # step still waits for its results on the host.
    graph = None
    try:
        body()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            body()
        graph = g
    except Exception as e:  # capture unsupported here: launch eagerly
        print(f"[bench] e2e graph capture failed ({e}); launching eagerly", file=sys.stderr)
        torch.cuda.synchronize()

    def step():
        if graph is not None:
            graph.replay()
        else:
            body()
        torch.cuda.current_stream().synchronize()

    out_len.zero_()
    for _ in range(2):
        step()
    out_len.zero_()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(job_throughput(b * B, world, ms / steps), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "launch": "cuda graph replay" if graph is not None else "eager"}


def load_traffic(kernel_class):
    """DRAM traffic per launch of a kernel class from the committed ncu summary, if it was
    captured from the current sources of that class's kernels."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        ent = d.get(kernel_class)
        if not ent:
            return None
        import hashlib
        for src, want in ent["sources"].items():
            with open(os.path.join(ROOT, src), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != want:
                    return None
        return ent["bytes_per_launch"]
    except Exception:
        return None


# ------------------------------------------------------------------ oracle (CPU) legs

def oracle_cycle(O, W, cfg, ctx, anchors, cu_s, st_s, taps_h, case, r, caches_by_req):
    """One request's cycle in the oracle: inject its new rows, draft its block, verify it."""
    lo, hi = int(cu_s[r]), int(cu_s[r + 1])
    T = int(ctx[r])
    c = O.context_features([t[lo:hi] for t in taps_h], W.mat("W_fc"), W.mat("g_ctx"), cfg.eps)
    pos = int(st_s[r]) + (torch.arange(hi - lo)).numpy()
    caches = caches_by_req[r]
    for l in range(cfg.L):
        K, V = O.inject_kv(c, pos, W.layer(l, "Wk"), W.layer(l, "Wv"), cfg.nkv, cfg.hd,
                           cfg.rope_base)
        caches[l][0][pos] = K
        caches[l][1][pos] = V
    toks, _ = O.draft_block(int(anchors[r]), T, [(k[:T], v[:T]) for k, v in caches], W, cfg)
    return O.verify_request(case["logits"][r], case["draft"][r])


def _oracle_caches(cfg, T, seed):
    import numpy as np

    rng = np.random.default_rng(seed)
    s = synth.gen.kv_std(cfg)
    return [(rng.normal(0, s, size=(T, cfg.nkv, cfg.hd)), rng.normal(0, s, size=(T, cfg.nkv, cfg.hd)))
            for _ in range(cfg.L)]


def cpu_baseline(w, cfg, ctx, anchors, cu_s, st_s, n_s, case, n_req=1):
    """The oracle, as it stands, on a bounded sample: the first request's full cycle."""
    import oracle as O

    taps_h = synth.make_tap_hiddens(cfg, n_s, label="taps_steady")
    caches = {r: _oracle_caches(cfg, int(ctx[r]), r) for r in range(n_req)}
    threads = torch.get_num_threads()
    t0 = time.perf_counter()
    W = O.Weights64(w, cfg)
    for r in range(n_req):
        oracle_cycle(O, W, cfg, ctx, anchors, cu_s, st_s, taps_h, case, r, caches)
    dt = time.perf_counter() - t0
    return {"value": round(n_req * cfg.B / dt, 4), "unit": UNIT, "cores": os.cpu_count(),
            "threads": threads, "kind": "oracle",
            "sample": f"{n_req} of {cfg.batch} requests: inject its rows, 2-step draft, verify; "
                      f"fp64 NumPy, weights converted once per sample ({dt:.1f} s)"}


def run_reference(args):
    """The oracle timed as the reference arm: each step is one request's cycle."""
    import oracle as O

    cfg = synth.get_config(WORKLOAD)
    w = synth.make_weights(cfg)
    ctx = synth.make_ctx_lens(cfg)
    anchors = synth.make_anchors(cfg)
    cu_s, st_s, n_s = synth.make_inject_layout(cfg, ctx, "steady")
    case = synth.make_verify_case(cfg.batch, cfg.B, cfg.V, "bench_ref", plant=cfg.plant)
    taps_h = synth.make_tap_hiddens(cfg, n_s, label="taps_steady")
    W = O.Weights64(w, cfg)
    caches = {r: _oracle_caches(cfg, int(ctx[r]), r) for r in range(cfg.batch)}
    times = []
    for i in range(args.warmup + args.steps):
        r = i % cfg.batch
        t0 = time.perf_counter()
        oracle_cycle(O, W, cfg, ctx, anchors, cu_s, st_s, taps_h, case, r, caches)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = cfg.B / sec
    cores = os.cpu_count()
    # n_gpus is the launch's N (the line pairs with our arm's line at that N); the
    # oracle itself runs on rank 0's host cores
    return {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
            "device": "cpu", "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random-init weights and inputs)", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one request's cycle per step"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores,
                             "kind": "oracle",
                             "sample": "one of 32 requests per step: inject, 2-step draft, verify"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ main

def prefill_report(cfg, n_rows, ms, peaks):
    """The timed prefill injection (every context position of every request): its two
    GEMMs (fc over the concatenated taps, the layer-batched K/V projection) dominate
    and are tensor-bound at this many rows."""
    kv = cfg.nkv * cfg.hd
    flops = 2 * n_rows * (cfg.d * cfg.n_tap * cfg.H_t + cfg.L * 2 * kv * cfg.d)
    tf = flops / (ms / 1e3) / 1e12
    # one call of tens of milliseconds right after an idle setup: the burst regime
    peak = peaks["bf16_tflops"]
    return {"rows": int(n_rows), "ms": round(ms, 3), "TFLOPs": round(tf, 1),
            "frac_tensor": round(tf / peak, 4), "peak_kind": "bf16 burst"}


def gemm_report():
    """Context for the projection GEMMs: the library's tcgen05 GEMM (through its test
    hook, with the split count and launch mode the draft path picks) next to
    torch.matmul (cuBLAS, not on the hot path) on the same fp16 shapes, one JSON line
    per shape. Each call runs on a freshly flushed L2; median of 15 calls."""
    import ctypes
    from block_diffusion_speculative_gemm_b200 import dflash as D

    dev = torch.device("cuda")
    cfg = synth.get_config(WORKLOAD)
    d, I, kv = cfg.d, cfg.I, cfg.nkv * cfg.hd
    qkv = cfg.nq * cfg.hd + 2 * kv
    M, n_inj = cfg.batch * cfg.B, 154
    shapes = [("qkv", qkv, d, M), ("o", d, cfg.nq * cfg.hd, M), ("gate_up", 2 * I, d, M),
              ("down", d, I, M), ("inject_fc", d, cfg.n_tap * cfg.H_t, n_inj),
              ("inject_kv", cfg.L * 2 * kv, d, n_inj)]
    L = D.lib()
    err = D.new_workspace(256)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream().cuda_stream

    def median_ms(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(15):
            flush.zero_()
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    for name, N, K, Mr in shapes:
        W = (torch.randn(N, K, device=dev) * 0.02).half()
        X = torch.randn(Mr, K, device=dev).half()
        Wt = D.debug_tile_weights(W)
        splits = L.dflash_debug_pick_splits(Mr, N, K)
        out = torch.empty(splits * Mr * N, device=dev)
        used = ctypes.c_int(0)

        def ours():
            r = L.dflash_debug_gemm_tiled(ctypes.c_void_p(Wt.data_ptr()), N, K,
                                          ctypes.c_void_p(X.data_ptr()), Mr, D.F16, splits,
                                          ctypes.c_void_p(out.data_ptr()), ctypes.byref(used),
                                          ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(st))
            assert r == 0, r

        t_ours = median_ms(ours)
        t_cublas = median_ms(lambda: torch.matmul(X, W.t()))
        print(json.dumps({"gemm": name, "N": N, "K": K, "M": Mr, "splits": splits,
                          "tcgen05_us": round(t_ours * 1e3, 1),
                          "cublas_us": round(t_cublas * 1e3, 1),
                          "tcgen05_TFLOPs": round(2 * Mr * N * K / t_ours / 1e9, 1),
                          "tcgen05_weight_GBps": round(N * K * 2 / t_ours / 1e6)}), flush=True)
        del W, Wt, X, out
    assert D.get_error(err) == 0


def graph_report():
    """One cycle (steady-state injection, the 2-step draft, verify) launched call by
    call versus replayed from a CUDA graph captured once, every cycle followed by a
    host wait for its results (as a serving loop reading its accepted tokens would),
    at batch 1, 8 and 32 of the 8B-shaped workload. One JSON line per batch."""
    from block_diffusion_speculative_gemm_b200 import dflash as D

    dev = torch.device("cuda")
    base = synth.get_config(WORKLOAD)
    B, V = base.B, base.V
    model = D.Model(base, to_device(synth.make_weights(base), dev),
                    base.cache_cap + 2 * B + 16)
    n = 50
    stream = torch.cuda.current_stream()
    for batch in (1, 8, 32):
        cfg = base.replace(batch=batch)
        ctx = synth.make_ctx_lens(cfg)
        anchors = synth.make_anchors(cfg).to(dev)
        cap = cfg.cache_cap
        kc = torch.zeros((cfg.L, batch, cfg.nkv, cap, cfg.hd), dtype=model.cache_dtype,
                         device=dev)
        vc = torch.zeros_like(kc)
        cu, st, n_rows = synth.make_inject_layout(cfg, ctx, "steady")
        taps = [t.to(dev) for t in synth.make_tap_hiddens(cfg, n_rows, label="graph_taps")]
        logits = synth.make_verify_case(batch, B, V, "graph", plant=cfg.plant)["logits"].to(dev)
        ws = D.new_workspace(max(model.workspace_size(batch, B, n_rows),
                                 D.verify_workspace_size(batch, B, V)))
        cu_d, st_d, ctx_d = cu.to(dev), st.to(dev), ctx.to(dev)
        draft = torch.zeros((batch, B), dtype=torch.int32, device=dev)
        out_tok = torch.zeros((batch, (2 * n + 16) * B), dtype=torch.int32, device=dev)
        out_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        seq = torch.zeros(batch, dtype=torch.int32, device=dev)
        acc = torch.zeros(batch, dtype=torch.int32, device=dev)
        nxt = torch.zeros(batch, dtype=torch.int32, device=dev)

        def cycle():
            D.inject_kv(model, taps, cu_d, st_d, kc, vc, ws)
            D.draft_block(model, anchors, ctx_d, kc, vc, B, cfg.steps, draft, ws)
            D.verify(logits, draft, out_tok, out_len, seq, acc, nxt, ws)

        def timed(fn):
            for _ in range(3):
                fn()
                stream.synchronize()
            out_len.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
                stream.synchronize()
            e1.record(stream)
            torch.cuda.synchronize()
            out_len.zero_()
            return e0.elapsed_time(e1) / n

        eager_ms = timed(cycle)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            cycle()
        graph_ms = timed(g.replay)
        assert D.get_error(ws) == 0
        print(json.dumps({"batch": batch, "block": B, "cycles": n,
                          "eager_ms_per_cycle": round(eager_ms, 4),
                          "graph_ms_per_cycle": round(graph_ms, 4),
                          "saving_ms": round(eager_ms - graph_ms, 4),
                          "graph_block_tok_s": round(batch * B / (graph_ms / 1e3), 1)}), flush=True)
        del kc, vc, ws, g
    model.close()


def sampled_verify_report():
    """Sampled (temperature) verify at the 8B-shaped batch (32 requests, block 8,
    vocabulary 151936, bf16 target and draft logits) against its HBM roofline, with
    greedy verify on the same target logits for context.  The algorithmic bytes
    are one read of the target rows (b*B*V*2) and of the draft rows 1..B-1
    (b*(B-1)*V*2); the draw's second read of one row pair per request is not
    counted.  Every iteration reads fresh logit buffers (two sets alternate, each
    larger than L2 together with the flush), and the L2 is flushed in between.
    One JSON line."""
    from block_diffusion_speculative_gemm_b200 import dflash as D

    peaks = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    dev = torch.device("cuda")
    b, B, V, tau = 32, 8, 151936, 1.0
    sets = []
    for k in range(2):
        c = synth.make_sampled_verify_case(b, B, V, f"bench_sv{k}", plant=("geometric", 4.0))
        sets.append((c["target"].to(dev), c["draft_logits"].to(dev), c["draft"].to(dev)))
    out = torch.zeros((b, 4096), dtype=torch.int32, device=dev)
    out_len = torch.zeros(b, dtype=torch.int32, device=dev)
    seq = torch.zeros(b, dtype=torch.int32, device=dev)
    acc = torch.zeros(b, dtype=torch.int32, device=dev)
    nxt = torch.zeros(b, dtype=torch.int32, device=dev)
    ws = D.new_workspace(max(D.verify_sampled_workspace_size(b, B, V),
                             D.verify_workspace_size(b, B, V)))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n=50):
        for k in range(5):
            fn(k)
        torch.cuda.synchronize()
        ts = []
        for k in range(n):
            out_len.zero_()
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(k)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    def sampled(k):
        Z, Y, d = sets[k % 2]
        D.verify_sampled(Z, Y, d, tau, 0x5EED, k, out, out_len, seq, acc, nxt, ws)

    def greedy(k):
        Z, _, d = sets[k % 2]
        D.verify(Z, d, out, out_len, seq, acc, nxt, ws)

    ms_s = timed(sampled)
    ms_g = timed(greedy)
    assert D.get_error(ws) == 0

    # context only (not on the path): PyTorch's row argmax over the same target
    # logits, the library reduction that reads the same bytes as greedy verify
    def torch_argmax(k):
        Z, _, _ = sets[k % 2]
        torch.argmax(Z.view(b * B, V), dim=-1)

    ms_t = timed(torch_argmax)
    bytes_s = b * (2 * B - 1) * V * 2
    bytes_g = b * B * V * 2
    print(json.dumps({
        "report": "sampled_verify", "workload": "qwen3_8b_bs32 verify (32 x 8 x 151936, bf16)",
        "temperature": tau, "sampled_us": round(ms_s * 1e3, 2),
        "sampled_algorithmic_GBps": round(bytes_s / ms_s / 1e6, 1),
        "sampled_frac_hbm": round(bytes_s / ms_s / 1e6 / hbm, 4),
        "greedy_us": round(ms_g * 1e3, 2),
        "greedy_frac_hbm": round(bytes_g / ms_g / 1e6 / hbm, 4),
        "torch_argmax_us": round(ms_t * 1e3, 2),
        "torch_argmax_frac_hbm": round(bytes_g / ms_t / 1e6 / hbm, 4),
        "rows_per_s_sampled": round(b * B / (ms_s / 1e3), 1),
        "hbm_peak_GBps": hbm, "peak_source": peaks["source"]}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dflash", choices=["dflash", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: override the draft layer count")
    ap.add_argument("--gemm-report", action="store_true",
                    help="context only: time the projection GEMMs against torch.matmul")
    ap.add_argument("--graph-report", action="store_true",
                    help="cycles launched call by call versus replayed from a CUDA graph")
    ap.add_argument("--sampled-verify-report", action="store_true",
                    help="sampled (temperature) verify against its HBM roofline")
    ap.add_argument("--attn-schedule", type=int, default=0,
                    help="tuning only: draft attention schedule (0 default grid, 1 persistent, "
                         "2 grid on the tcgen05 kernel)")
    args = ap.parse_args()
    if args.gemm_report:
        gemm_report()
        return
    if args.graph_report:
        graph_report()
        return
    if args.sampled_verify_report:
        sampled_verify_report()
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_dflash(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
