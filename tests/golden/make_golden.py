"""Writes tests/golden/tiny_f32_oracle.json and sampled_oracle.json from the oracle alone.

Run from the repository root: ``python tests/golden/make_golden.py``.  It
imports only ``oracle`` and the seeded input generators in ``synth``; the
stored values are a regression guard for the oracle itself.
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle as O  # noqa: E402
import synth  # noqa: E402


def tiny_case():
    cfg = synth.get_config("tiny_f32")
    w = synth.make_weights(cfg)
    W = O.Weights64(w, cfg)
    T = cfg.ctx[1]
    taps = synth.make_tap_hiddens(cfg, T)
    cu = np.array([0, T])
    st = np.array([0])
    inj = O.inject_kv_requests(taps, cu, st, W, cfg)
    caches = [(inj[(l, 0)][1], inj[(l, 0)][2]) for l in range(cfg.L)]
    anchor = int(synth.make_anchors(cfg)[0])
    toks, rec = O.draft_block(anchor, T, caches, W, cfg)
    case = synth.make_verify_case(1, cfg.B, cfg.V, "golden", plant=cfg.plant, dtype="f32")
    vr = O.verify_batch(case["logits"], case["draft"], np.zeros((1, 16)), np.zeros(1), 16,
                        np.array([T]))
    return {
        "config": cfg.name,
        "anchor": anchor,
        "draft_tokens": [int(t) for t in toks],
        "draft_margins": [float(m) for m in rec[0]["stats"]["margin"]],
        "k_cache_l0_pos5_head0": [float(v) for v in caches[0][0][5, 0, :8]],
        "verify_accept": int(vr["accept"][0]),
        "verify_emitted": [int(t) for t in vr["out_tokens"][0, :int(vr["out_len"][0])]],
    }


def sampled_case():
    """Sampled verify on a small batch and sampled drafting on the tiny model."""
    b, B, V, tau, seed, offset = 4, 6, 300, 0.8, 0x5EED, 3
    c = synth.make_sampled_verify_case(b, B, V, "golden_sv", plant=("geometric", 4.0),
                                       dtype="f32")
    res = O.sampled_verify.sampled_verify_batch(c["target"], c["draft_logits"], c["draft"], tau,
                                                seed, offset, np.zeros((b, 3 * B)),
                                                np.zeros(b), 3 * B, np.zeros(b))
    cfg = synth.get_config("tiny_f32")
    W = O.Weights64(synth.make_weights(cfg), cfg)
    T = cfg.ctx[1]
    taps = synth.make_tap_hiddens(cfg, T)
    inj = O.inject_kv_requests(taps, np.array([0, T]), np.array([0]), W, cfg)
    caches = [(inj[(l, 0)][1], inj[(l, 0)][2]) for l in range(cfg.L)]
    toks, q, rec = O.sampled_draft.sampled_draft_block(5, T, caches, W, cfg, 0.9, seed, offset, 0,
                                                       steps=2)
    return {
        "verify_accept": [int(a) for a in res["accept"]],
        "verify_next_anchor": [int(t) for t in res["next_anchor"]],
        "verify_log_rho_first": [float(d["log_rho"][0]) for d in res["detail"]],
        "draft_tokens": [int(t) for t in toks],
        "draft_commit": [r["commit"] for r in rec],
        "draft_conf_step0": [float(x) for x in rec[0]["conf"]],
    }


if __name__ == "__main__":
    out = tiny_case()
    with open(os.path.join(HERE, "tiny_f32_oracle.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))
    out = sampled_case()
    with open(os.path.join(HERE, "sampled_oracle.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))
