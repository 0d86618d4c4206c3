"""Seeded generators.  Random numbers and workload structure only.

All tensors are created on the host (CPU) with ``torch.Generator`` seeded from
``sub_seed(master, labels...)``, so that any consumer regenerates identical
values from the same labels.
"""

from __future__ import annotations

import math
import zlib
from typing import Dict, List, Optional

import torch

from .configs import DraftConfig

MASTER_SEED = 0x5EED
_CHUNK = 1 << 25  # elements per generation chunk (keeps fp32 temporaries small)


def sub_seed(master: int, *labels) -> int:
    """A stable 63-bit seed derived from a master seed and a tuple of labels."""
    h = zlib.crc32(("|".join(str(x) for x in labels)).encode()) & 0xFFFFFFFF
    h2 = zlib.crc32(("#" + "|".join(str(x) for x in labels[::-1])).encode()) & 0xFFFFFFFF
    return ((int(master) * 0x9E3779B1) ^ (h << 31) ^ h2) & 0x7FFFFFFFFFFFFFFF


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def _dtype(cfg_or_str) -> torch.dtype:
    s = cfg_or_str if isinstance(cfg_or_str, str) else cfg_or_str.dtype
    return {"f32": torch.float32, "bf16": torch.bfloat16}[s]


def _randn(shape, std: float, seed: int, dtype: torch.dtype) -> torch.Tensor:
    """N(0, std^2) rounded to ``dtype``, generated in row chunks."""
    g = _gen(seed)
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        flat[s:e] = (torch.randn(e - s, generator=g) * std).to(dtype)
    return out


def _gain(cfg: DraftConfig, n: int, seed: int, dtype) -> torch.Tensor:
    if cfg.gain_std == 0.0:
        return torch.ones(n, dtype=dtype)
    g = _gen(seed)
    return (1.0 + cfg.gain_std * torch.randn(n, generator=g)).to(dtype)


def make_weights(cfg: DraftConfig, master: int = MASTER_SEED) -> Dict:
    """Random-init draft weights, all matrices in [out_features, in_features] layout.

    Keys: emb [V,d], W_fc [d, n_tap*H_t], g_ctx [d], layers (list of dicts with
    g_in, Wq [nq*hd,d], Wk [nkv*hd,d], Wv [nkv*hd,d], Wo [d,nq*hd], g_post,
    Wg [I,d], Wu [I,d], Wd [d,I]), g_final [d], W_lm [V,d].
    """
    dt = _dtype(cfg)
    s = lambda *lab: sub_seed(master, cfg.name, "w", *lab)
    w = {
        "emb": _randn((cfg.V, cfg.d), cfg.w_std, s("emb"), dt),
        "W_fc": _randn((cfg.d, cfg.n_tap * cfg.H_t), cfg.w_std, s("fc"), dt),
        "g_ctx": _gain(cfg, cfg.d, s("g_ctx"), dt),
        "g_final": _gain(cfg, cfg.d, s("g_final"), dt),
        "W_lm": _randn((cfg.V, cfg.d), cfg.w_std, s("lm"), dt),
        "layers": [],
    }
    for l in range(cfg.L):
        w["layers"].append({
            "g_in": _gain(cfg, cfg.d, s(l, "g_in"), dt),
            "Wq": _randn((cfg.nq * cfg.hd, cfg.d), cfg.w_std, s(l, "q"), dt),
            "Wk": _randn((cfg.nkv * cfg.hd, cfg.d), cfg.w_std, s(l, "k"), dt),
            "Wv": _randn((cfg.nkv * cfg.hd, cfg.d), cfg.w_std, s(l, "v"), dt),
            "Wo": _randn((cfg.d, cfg.nq * cfg.hd), cfg.w_std, s(l, "o"), dt),
            "g_post": _gain(cfg, cfg.d, s(l, "g_post"), dt),
            "Wg": _randn((cfg.I, cfg.d), cfg.w_std, s(l, "g"), dt),
            "Wu": _randn((cfg.I, cfg.d), cfg.w_std, s(l, "u"), dt),
            "Wd": _randn((cfg.d, cfg.I), cfg.w_std, s(l, "dn"), dt),
        })
    return w


def make_tap_hiddens(cfg: DraftConfig, n_rows: int, label: str = "taps",
                     master: int = MASTER_SEED) -> List[torch.Tensor]:
    """``n_tap`` tensors of tapped target hidden states, each [n_rows, H_t]."""
    dt = _dtype(cfg)
    return [_randn((n_rows, cfg.H_t), cfg.h_std, sub_seed(master, cfg.name, label, i), dt)
            for i in range(cfg.n_tap)]


def make_ctx_lens(cfg: DraftConfig, master: int = MASTER_SEED) -> torch.Tensor:
    """Per-request context length T_r (int32 [batch])."""
    if cfg.ctx[0] == "fixed":
        return torch.full((cfg.batch,), cfg.ctx[1], dtype=torch.int32)
    lo, hi = cfg.ctx[1], cfg.ctx[2]
    g = _gen(sub_seed(master, cfg.name, "ctx"))
    return torch.randint(lo, hi + 1, (cfg.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def make_anchors(cfg: DraftConfig, label: str = "anchor", master: int = MASTER_SEED) -> torch.Tensor:
    """Anchor token per request, uniform over the vocabulary minus the mask id."""
    g = _gen(sub_seed(master, cfg.name, label))
    return torch.randint(0, cfg.V - 1, (cfg.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def kv_std(cfg: DraftConfig) -> float:
    """Spread of an injected K/V entry: unit-rms features times a std-w_std projection."""
    return cfg.w_std * math.sqrt(cfg.d)


def make_kv_cache(cfg: DraftConfig, cap: Optional[int] = None, label: str = "kv",
                  master: int = MASTER_SEED, dtype: Optional[torch.dtype] = None):
    """Synthetic K/V cache contents [L, batch, nkv, cap, hd] (every slot filled),
    rounded to ``dtype`` (default: the workload's dtype)."""
    cap = cfg.cache_cap if cap is None else cap
    dt = _dtype(cfg) if dtype is None else dtype
    shp = (cfg.L, cfg.batch, cfg.nkv, cap, cfg.hd)
    k = _randn(shp, kv_std(cfg), sub_seed(master, cfg.name, label, "k"), dt)
    v = _randn(shp, kv_std(cfg), sub_seed(master, cfg.name, label, "v"), dt)
    return k, v


def sample_plants(plant, n: int, B: int, seed: int) -> torch.Tensor:
    """Planted accept lengths in [0, B-1]: uniform, or geometric(mean) capped at B-1."""
    g = _gen(seed)
    if plant[0] == "uniform":
        return torch.randint(0, B, (n,), generator=g, dtype=torch.int64)
    mean = float(plant[1])
    p = 1.0 / (1.0 + mean)
    u = torch.rand(n, generator=g, dtype=torch.float64).clamp_min(1e-300)
    k = torch.floor(torch.log(u) / math.log(1.0 - p)).to(torch.int64)
    return k.clamp(0, B - 1)


def make_inject_layout(cfg: DraftConfig, ctx_lens: torch.Tensor, mode: str,
                       master: int = MASTER_SEED):
    """Rows to inject per request.

    ``prefill``: every context position 0..T_r-1.  ``steady``: the a+1 rows
    accepted in the previous cycle, i.e. positions [T_r - n_r, T_r) with
    n_r - 1 drawn from the workload's planted accept-length distribution.
    Returns (cu_rows int32 [batch+1], start_pos int32 [batch], n_rows).
    """
    b = cfg.batch
    if mode == "prefill":
        n = ctx_lens.to(torch.int64)
        start = torch.zeros(b, dtype=torch.int64)
    elif mode == "steady":
        a = sample_plants(cfg.plant, b, cfg.B, sub_seed(master, cfg.name, "steady"))
        n = torch.minimum(a + 1, ctx_lens.to(torch.int64))
        start = ctx_lens.to(torch.int64) - n
    else:
        raise ValueError(mode)
    cu = torch.zeros(b + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(n, 0)
    return cu.to(torch.int32), start.to(torch.int32), int(cu[-1])


def _bf16_step(x: torch.Tensor, up: bool) -> torch.Tensor:
    """Next representable bf16 value above (up) or below a bf16 tensor (finite, nonzero)."""
    bits = x.view(torch.int16).to(torch.int32)
    pos = bits >= 0
    delta = torch.where(pos == up, torch.ones_like(bits), -torch.ones_like(bits))
    return (bits + delta).to(torch.int16).view(torch.bfloat16)


def make_verify_case(b: int, B: int, V: int, label: str, plant=("uniform",), dtype: str = "bf16",
                     adversarial: bool = False, raise_by: float = 8.0, master: int = MASTER_SEED,
                     draft: Optional[torch.Tensor] = None):
    """Target logits [b, B, V] ~ N(0,1) with planted accept prefixes.

    Draft tokens are uniform over the vocabulary unless ``draft`` supplies
    them (e.g. a drafted block the logits should partly agree with).  For rows i < a_r the draft
    token d[i+1] gets its logit raised by ``raise_by``; at row a_r (if a_r < B-1)
    d[a_r+1] is lowered to the row minimum.  With ``adversarial`` some planted
    rows instead put d[i+1] one bf16 ulp above or below the row maximum, or
    exactly equal to it next to another copy of the maximum at a lower or
    higher index.  The accept length the rule produces is decided by the
    oracle, not by this generator.
    """
    seed = sub_seed(master, "verify", label, b, B, V)
    g = _gen(seed)
    dt = _dtype(dtype)
    logits = torch.randn((b, B, V), generator=g).to(dt)
    rnd = torch.randint(0, V, (b, B), generator=g, dtype=torch.int64).to(torch.int32)
    draft = rnd if draft is None else draft.to(torch.int32).cpu().clone()
    plants = sample_plants(plant, b, B, sub_seed(seed, "plant"))
    modes = torch.randint(0, 5, (b, B), generator=g)
    others = torch.randint(0, V, (b, B), generator=g)
    for r in range(b):
        a = int(plants[r])
        for i in range(B - 1):
            t = int(draft[r, i + 1])
            row = logits[r, i]
            if i < a:
                m = int(modes[r, i]) if adversarial else 0
                if m == 0:
                    row[t] = (row[t].float() + raise_by).to(dt)
                elif dt == torch.bfloat16 and m in (1, 2):
                    mx = row.max()
                    row[t] = _bf16_step(mx.reshape(1), up=(m == 1))[0] if mx != 0 else mx
                else:
                    mx = row.max()
                    row[t] = mx
                    row[int(others[r, i])] = mx
            elif i == a:
                row[t] = row.min()
    return {"logits": logits, "draft": draft, "planted": plants.to(torch.int32)}


def make_sampled_verify_case(b: int, B: int, V: int, label: str, plant=("uniform",),
                             dtype: str = "bf16", raise_target: float = 6.0,
                             raise_draft: float = 6.0, master: int = MASTER_SEED):
    """Target logits Z and draft logits Y, both [b, B, V] ~ N(0,1), with draft tokens.

    Draft tokens are uniform over the vocabulary (column 0 is the anchor).  For
    every block position j >= 1 the draft's own logit Y[r, j, d_j] is raised by
    ``raise_draft`` (the draft favours what it proposed); for target rows
    i < a_r the target logit Z[r, i, d_{i+1}] is raised by ``raise_target``
    (planted agreement).  Row 0 of Y is drawn but unused.  What sampled
    verification accepts is decided by the oracle, not by this generator.
    """
    seed = sub_seed(master, "sampled_verify", label, b, B, V)
    g = _gen(seed)
    dt = _dtype(dtype)
    Z = torch.randn((b, B, V), generator=g)
    Y = torch.randn((b, B, V), generator=g)
    draft = torch.randint(0, V, (b, B), generator=g, dtype=torch.int64)
    plants = sample_plants(plant, b, B, sub_seed(seed, "plant"))
    rows = torch.arange(b)
    for j in range(1, B):
        Y[rows, j, draft[:, j]] += raise_draft
    for i in range(B - 1):
        sel = plants > i
        Z[rows[sel], i, draft[sel, i + 1]] += raise_target
    return {"target": Z.to(dt), "draft_logits": Y.to(dt), "draft": draft.to(torch.int32),
            "planted": plants.to(torch.int32)}
