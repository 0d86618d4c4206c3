"""Seeded synthetic inputs for the DFlash draft hot path.

This module is shared by the tests, the benchmark and the oracle checks. It
draws random numbers and shapes them into workloads (weights, tapped hidden
states, context lengths, KV-cache contents, target logits with planted
accept lengths). It holds none of the method's arithmetic: no projection,
normalisation, attention, argmax or acceptance rule lives here.

Every tensor is produced on the host with a seeded ``torch.Generator`` so the
CPU oracle and the GPU path read bit-identical values.
"""

from .configs import CONFIGS, DraftConfig, VERIFY_SWEEP, get_config
from .gen import (
    sub_seed,
    make_weights,
    make_tap_hiddens,
    make_ctx_lens,
    make_anchors,
    make_kv_cache,
    make_verify_case,
    make_sampled_verify_case,
    make_inject_layout,
)

__all__ = [
    "CONFIGS",
    "DraftConfig",
    "VERIFY_SWEEP",
    "get_config",
    "sub_seed",
    "make_weights",
    "make_tap_hiddens",
    "make_ctx_lens",
    "make_anchors",
    "make_kv_cache",
    "make_verify_case",
    "make_sampled_verify_case",
    "make_inject_layout",
]
