"""The benchmark's roofline arithmetic against closed forms of the workload.

`bench.step_algorithmic` gives the algorithmic bytes and flops that every
reported roofline fraction divides by.  Here they are rebuilt from the shapes
alone and checked against the per-cycle budget of the 8B-shaped workload:

* draft layer weights: 1.929 GB per denoising step;
* LM head: 1.245 GB per step;
* injection weights: 251.7 MB;
* verify logits: 77.8 MB;
* context K/V: 4096 B per token per layer.
"""

import pytest

import bench
import synth

PEAKS = {"hbm_gbs": 6550.4, "bf16_tflops": 1644.9, "bf16_tflops_sustained": 1403.3}


@pytest.fixture(scope="module")
def cyc():
    cfg = synth.get_config("qwen3_8b_bs32")
    ctx = synth.make_ctx_lens(cfg)
    _, _, n = synth.make_inject_layout(cfg, ctx, "steady")
    return cfg, ctx, n, bench.step_algorithmic(cfg, n, ctx, PEAKS)


def test_weight_bytes_match_the_budget(cyc):
    cfg, ctx, n, out = cyc
    d, q, kv, I = cfg.d, cfg.nq * cfg.hd, cfg.nkv * cfg.hd, cfg.I
    layer_w = (q + 2 * kv) * d + d * q + 2 * I * d + d * I  # elements per layer
    assert abs(cfg.L * layer_w * 2 - 1.929e9) < 1e6
    assert abs(cfg.V * d * 2 - 1.2447e9) < 1e6
    inject_w = d * cfg.n_tap * cfg.H_t + cfg.L * 2 * kv * d
    assert abs(inject_w * 2 - 251.7e6) < 1e5
    # the GEMM class: weights once per step (and the injection's once), plus
    # activations in and out
    M = cfg.batch * cfg.B
    act = 0
    for N, K in ((q + 2 * kv, d), (d, q), (2 * I, d), (d, I)):
        act += cfg.L * (M * K * 2 + M * N * 2)
    inj_act = n * cfg.n_tap * cfg.H_t * 2 + n * d * 2 + n * d * 2 + n * cfg.L * 2 * kv * 2
    want = cfg.steps * (cfg.L * layer_w * 2 + act) + inject_w * 2 + inj_act
    assert out["gemm"]["bytes"] == want


def test_lm_head_verify_and_attention_bytes(cyc):
    cfg, ctx, n, out = cyc
    b, B, V, d = cfg.batch, cfg.B, cfg.V, cfg.d
    tiles = -(-V // 128)
    rows = [b * (B - 1)]
    rem = B - 1
    for t in range(cfg.steps - 1):
        rem -= -(-rem // (cfg.steps - t))
        rows.append(b * rem)
    want_lm = sum(V * d * 2 + r * d * 2 + r * tiles * 16 for r in rows)
    assert out["lm_head"]["bytes"] == want_lm
    assert rows == [224, 96]  # the two denoising steps' masked rows at this workload
    assert out["verify"]["bytes"] == b * B * V * 2 + b * B * 8
    assert abs(b * B * V * 2 - 77.8e6) < 0.1e6
    kv_per_token_layer = cfg.nkv * cfg.hd * 2 * 2
    assert kv_per_token_layer == 4096
    T = int(ctx.sum())
    block = b * B * (2 * cfg.nq * cfg.hd + 2 * cfg.nkv * cfg.hd) * 2
    assert out["attention"]["bytes"] == cfg.steps * cfg.L * (T * kv_per_token_layer + block)


def test_roofline_times_are_the_slower_resource(cyc):
    cfg, ctx, n, out = cyc
    hbm, tc = PEAKS["hbm_gbs"] * 1e9, PEAKS["bf16_tflops_sustained"] * 1e12
    for k in ("attention", "verify"):
        assert out[k]["roof_s"] == pytest.approx(out[k]["bytes"] / hbm, rel=1e-12)
    # a GEMM class roof is at least each of its two bounds taken over the class
    for k in ("gemm", "lm_head"):
        c = out[k]
        assert c["roof_s"] >= c["bytes"] / hbm * (1 - 1e-12)
        assert c["roof_s"] >= c["flops"] / tc * (1 - 1e-12)
        assert c["flops"] > 0
    M = cfg.batch * cfg.B
    d, q, kv, I = cfg.d, cfg.nq * cfg.hd, cfg.nkv * cfg.hd, cfg.I
    fl = cfg.steps * cfg.L * 2 * M * ((q + 2 * kv) * d + d * q + 2 * I * d + d * I)
    fl += 2 * n * (d * cfg.n_tap * cfg.H_t + cfg.L * 2 * kv * d)
    assert out["gemm"]["flops"] == fl
    total_ms = sum(c["roof_s"] for c in out.values()) * 1e3
    assert 1.4 < total_ms < 1.8  # the cycle roofline quoted with the bench (1.595 ms)


def test_tensor_peak_follows_the_sampled_clock():
    # near max clock: the burst figure; a clock lowered by the power cap: sustained
    assert bench.tensor_peak(PEAKS, {"sm_mhz": 1897.5, "sm_max_mhz": 1965.0}) == (1644.9, "burst")
    assert bench.tensor_peak(PEAKS, {"sm_mhz": 1350.0, "sm_max_mhz": 1965.0}) == (
        1403.3, "sustained")
    # no clock samples: the conservative sustained figure
    assert bench.tensor_peak(PEAKS, {"sm_mhz": None, "sm_max_mhz": None})[1] == "sustained"
    # no sustained figure measured: burst
    assert bench.tensor_peak({"bf16_tflops": 1590.0}, {})[1] == "burst"
