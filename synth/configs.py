"""Workload shapes for the DFlash draft hot path.

Shapes follow the workloads described for DFlash-style drafting: a draft with
five layers on top of a Qwen3-shaped target ("DFlash + Spec V2 深度解析",
§4.2 训练配置 gives five draft layers, block 8 and two diffusion steps;
§2.3 块扩散 gives block sizes 4/8/16; "DFlash: Block Diffusion for Flash
Speculative Decoding", §Spec V2 引擎优化 quotes a Qwen3-8B target on one B200
at concurrency 32).  The pages print no model dimensions, so the Qwen3-4B and
Qwen3-8B hidden sizes, head counts, MLP widths and vocabulary are the public
model cards' figures.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple


@dataclass(frozen=True)
class DraftConfig:
    name: str
    dtype: str            # storage/compute type of weights and activations: "f32" or "bf16"
    H_t: int              # target hidden size (per tapped layer)
    n_tap: int            # number of tapped target layers
    L: int                # draft layers
    d: int                # draft hidden size
    nq: int               # query heads
    nkv: int              # key/value heads
    hd: int               # head dim
    I: int                # SwiGLU intermediate size
    V: int                # vocabulary
    batch: int
    ctx: Tuple            # ("fixed", T) or ("uniform", lo, hi)
    B: int                # block size
    steps: int            # denoising steps
    plant: Tuple          # ("uniform",) or ("geometric", mean)
    eps: float = 1e-6
    rope_base: float = 1e6
    w_std: float = 0.02
    h_std: float = 0.02
    gain_std: float = 0.0  # 0 -> unit gains

    @property
    def mask_id(self) -> int:
        return self.V - 1

    @property
    def max_ctx(self) -> int:
        return self.ctx[1] if self.ctx[0] == "fixed" else self.ctx[2]

    @property
    def cache_cap(self) -> int:
        # room for the longest context, one block and one more cycle of accepted tokens
        c = self.max_ctx + 2 * self.B
        return (c + 15) // 16 * 16

    @property
    def qkv_out(self) -> int:
        return (self.nq + 2 * self.nkv) * self.hd

    def replace(self, **kw) -> "DraftConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # correctness-only tiny draft, fp32 storage
    "tiny_f32": DraftConfig(
        name="tiny_f32", dtype="f32", H_t=256, n_tap=3, L=2, d=256, nq=4, nkv=2, hd=64,
        I=512, V=1024, batch=1, ctx=("fixed", 128), B=4, steps=1, plant=("uniform",)),
    # Qwen3-4B-shaped draft, one request (stands in for concurrency-1 serving)
    "qwen3_4b_bs1": DraftConfig(
        name="qwen3_4b_bs1", dtype="bf16", H_t=2560, n_tap=5, L=5, d=2560, nq=32, nkv=8,
        hd=128, I=9728, V=151936, batch=1, ctx=("fixed", 2048), B=16, steps=1,
        plant=("geometric", 3.5)),
    # Qwen3-8B-shaped draft, 32 requests (stands in for concurrency-32 serving)
    "qwen3_8b_bs32": DraftConfig(
        name="qwen3_8b_bs32", dtype="bf16", H_t=4096, n_tap=5, L=5, d=4096, nq=32, nkv=8,
        hd=128, I=12288, V=151936, batch=32, ctx=("uniform", 512, 4096), B=8, steps=2,
        plant=("geometric", 4.0)),
    # long context, same 8B shape: 4 requests x 32768 tokens, block 16
    "qwen3_8b_ctx32k": DraftConfig(
        name="qwen3_8b_ctx32k", dtype="bf16", H_t=4096, n_tap=5, L=5, d=4096, nq=32,
        nkv=8, hd=128, I=12288, V=151936, batch=4, ctx=("fixed", 32768), B=16, steps=1,
        plant=("geometric", 4.0)),
}

# verify-only sweep: batch x block x vocab 151936, bf16 logits N(0,1)
VERIFY_SWEEP = {
    "batches": (1, 8, 32, 128),
    "blocks": (4, 8, 16),
    "V": 151936,
}


def get_config(key: str, **overrides) -> DraftConfig:
    cfg = CONFIGS[key]
    return cfg.replace(**overrides) if overrides else cfg


def shrink(cfg: DraftConfig, *, L: Optional[int] = None, V: Optional[int] = None,
           batch: Optional[int] = None, ctx: Optional[Tuple] = None, I: Optional[int] = None,
           d: Optional[int] = None, H_t: Optional[int] = None) -> DraftConfig:
    """A smaller variant of a workload with the same head geometry (for fast parity)."""
    kw = {}
    for k, v in (("L", L), ("V", V), ("batch", batch), ("ctx", ctx), ("I", I), ("d", d),
                 ("H_t", H_t)):
        if v is not None:
            kw[k] = v
    return cfg.replace(name=cfg.name + "_small", **kw)
