"""Helpers for the GPU parity tests: build models from seeded weights and
compare library results with the fp64 oracle under the stated tolerances.

Tolerances (the draft-path rules for bf16 storage with fp32 accumulation):
  * K/V cache entries and LM-head logits: max |gpu - oracle| <= 1e-2 * max |oracle|
    per compared tensor;
  * draft tokens: identical to the oracle's argmax except where the oracle's
    top-2 logit margin is below 0.05 (counted);
  * commit sets (s > 1 steps): the oracle's choice, or another size-k set that
    differs from it only among positions whose confidences are within 5%
    (relative) of each other (counted).  The next step then continues from the
    set and tokens the oracle itself admitted.
  * verify: bit-exact.
"""


import numpy as np
import torch

import oracle as O
import synth
from synth.device import to_device
from block_diffusion_speculative_gemm_b200 import dflash as D

REL_TOL = 1e-2
MARGIN_BAND = 0.05
CONF_BAND = 0.05

_MODELS = {}


def max_pos_for(cfg, cap=None):
    cap = cfg.cache_cap if cap is None else cap
    return cap + 2 * cfg.B + 16


class Built:
    """Host weights, their oracle view, device copies and the library model."""

    def __init__(self, cfg, cap=None):
        self.cfg = cfg
        self.cap = cfg.cache_cap if cap is None else cap
        self.w = synth.make_weights(cfg)
        self.W = O.Weights64(self.w, cfg)
        self.wd = to_device(self.w)
        self.model = D.Model(cfg, self.wd, max_pos_for(cfg, self.cap))

    def tdtype(self):
        return torch.bfloat16 if self.cfg.dtype == "bf16" else torch.float32


def built(cfg, cap=None) -> Built:
    key = (cfg, cap)
    if key not in _MODELS:
        _MODELS.clear()  # keep at most one model resident
        torch.cuda.empty_cache()
        _MODELS[key] = Built(cfg, cap)
    return _MODELS[key]


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0))


# Per-test parity figures (near-tie counts, largest relative errors) collected
# during a run; tests/conftest.py writes them as JSON at the end of the session
# when DFLASH_PARITY_RECORD names a file.
RECORD = {}


def record(test: str, **fields):
    ent = RECORD.setdefault(test, {})
    for k, v in fields.items():
        if isinstance(v, (int, float)) and k.startswith("max_") and k in ent:
            ent[k] = max(ent[k], v)
        elif isinstance(v, int) and k in ent and not k.startswith("max_"):
            ent[k] += v
        else:
            ent[k] = v


class DraftReport:
    def __init__(self):
        self.token_near_ties = 0
        self.commit_near_ties = 0
        self.positions = 0
        self.max_logit_rel = 0.0

    def save(self, test: str, **extra):
        """Adds this report's counts to the session's parity record under `test`."""
        record(test, positions=self.positions, token_near_ties=self.token_near_ties,
               commit_near_ties=self.commit_near_ties, max_logit_rel=self.max_logit_rel,
               **extra)
        return self

    def __repr__(self):
        return (f"positions={self.positions} token_near_ties={self.token_near_ties} "
                f"commit_near_ties={self.commit_near_ties} max_logit_rel={self.max_logit_rel:.3e}")


def check_draft_request(b: Built, r: int, anchor: int, T: int, caches, gpu_tokens, gpu_cstep,
                        gpu_logits, steps: int, rep: DraftReport):
    """Walks the oracle through the denoising steps of request r, admitting the
    GPU's commit set / tokens only where the oracle's own near-tie bands allow.

    gpu_logits: per step, dict position -> fp32 logits row (or None)."""
    cfg = b.cfg
    B = cfg.B
    tokens = np.full(B, cfg.mask_id, dtype=np.int64)
    tokens[0] = anchor
    assert int(gpu_tokens[0]) == anchor
    masked = list(range(1, B))
    for t in range(steps):
        st = O.draft_step([tokens], [masked], [T], [caches], b.W, cfg,
                          keep_logits=gpu_logits is not None)[0]
        if gpu_logits is not None:
            for i, p in enumerate(st["pos"]):
                e = rel_err(gpu_logits[t][p], st["logits"][i])
                rep.max_logit_rel = max(rep.max_logit_rel, e)
                assert e <= REL_TOL, f"req {r} step {t} pos {p}: logits rel err {e:.3e}"
        k = O.commit_count(len(masked), steps - t)
        gpu_commit = sorted(p for p in masked if int(gpu_cstep[p]) == t)
        assert len(gpu_commit) == k, f"req {r} step {t}: committed {gpu_commit}, expected {k}"
        exact = O.select_commits(st["pos"], st["conf"], k)
        if gpu_commit != exact:
            valid = O.valid_commit_sets(st["pos"], st["conf"], k, CONF_BAND)
            assert gpu_commit in valid, (
                f"req {r} step {t}: commit {gpu_commit} not admitted (oracle {exact}, "
                f"conf {dict(zip(st['pos'], np.round(st['conf'], 6)))})")
            rep.commit_near_ties += 1
        for p in gpu_commit:
            i = st["pos"].index(p)
            g = int(gpu_tokens[p])
            rep.positions += 1
            if g != int(st["tok"][i]):
                assert st["margin"][i] < MARGIN_BAND and g in set(int(c) for c in st["cand"][i]), (
                    f"req {r} step {t} pos {p}: token {g} vs oracle {int(st['tok'][i])} "
                    f"(margin {st['margin'][i]:.4f})")
                rep.token_near_ties += 1
            tokens[p] = g
        masked = [p for p in masked if p not in gpu_commit]
    assert not masked


def oracle_caches_from(k_cache, v_cache, l_count, r, T):
    """Oracle view of request r's first T cache positions, per layer (float64)."""
    out = []
    for l in range(l_count):
        K = O.as_f64(k_cache[l, r, :, :T, :]).transpose(1, 0, 2)
        V = O.as_f64(v_cache[l, r, :, :T, :]).transpose(1, 0, 2)
        out.append((K, V))
    return out
