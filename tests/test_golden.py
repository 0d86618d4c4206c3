"""Golden fixtures: page facts (cited) and the oracle's own regression record."""

import json
import os

import pytest

import synth
from tests.golden.make_golden import sampled_case, tiny_case

G = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(G, name)) as f:
        return json.load(f)


def test_workloads_use_the_pages_block_sizes_and_layers():
    facts = _load("page_facts.json")
    for cfg in synth.CONFIGS.values():
        assert cfg.B in facts["block_sizes"]["value"]
        if cfg.L > 2:
            assert cfg.L == facts["draft_layers"]["value"]
    b8 = [c for c in synth.CONFIGS.values() if c.B == facts["training_block_and_steps"]["value"]["block"]]
    assert all(c.steps == facts["training_block_and_steps"]["value"]["diffusion_steps"] for c in b8)
    assert all(c.B in synth.VERIFY_SWEEP["blocks"] for c in synth.CONFIGS.values())


@pytest.mark.parametrize("name", ["qwen3_4b_bs1", "qwen3_8b_bs32"])
def test_planted_accept_lengths_sit_in_the_acceptable_band(name):
    # mean accepted tokens per block of the planted distribution (capped geometric)
    cfg = synth.get_config(name)
    band = _load("page_facts.json")["acceptance_length_bands"]["value"]
    a = synth.gen.sample_plants(cfg.plant, 200000, cfg.B, 1).double().mean().item()
    assert band["acceptable"] <= a <= band["excellent"] + 0.5


def test_oracle_regression_record():
    want = _load("tiny_f32_oracle.json")
    got = tiny_case()
    assert got["draft_tokens"] == want["draft_tokens"]
    assert got["verify_accept"] == want["verify_accept"]
    assert got["verify_emitted"] == want["verify_emitted"]
    assert got["draft_margins"] == pytest.approx(want["draft_margins"], rel=1e-12)
    assert got["k_cache_l0_pos5_head0"] == pytest.approx(want["k_cache_l0_pos5_head0"], rel=1e-12)


def test_sampled_oracle_regression_record():
    want = _load("sampled_oracle.json")
    got = sampled_case()
    for k in ("verify_accept", "verify_next_anchor", "draft_tokens", "draft_commit"):
        assert got[k] == want[k], k
    assert got["verify_log_rho_first"] == pytest.approx(want["verify_log_rho_first"], rel=1e-12)
    assert got["draft_conf_step0"] == pytest.approx(want["draft_conf_step0"], rel=1e-12)
