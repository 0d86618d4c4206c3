"""Per-entry sampling arithmetic of the draw kernels against float64.

The sampled verify and sampled drafting kernels score every vocabulary entry
with a Gumbel variate in log2 units, -log2(-ln U'), built from the hardware
base-2 logarithm and a short atanh series, and the residual draw weights with
log2(1 - 2^d) from the hardware exp2 / log2 and an expm1 series.  Their error
bounds (stated beside the functions) are checked here over random and edge
inputs through dflash_debug_sample_math, against the oracle's exact
exponential variates (pinned against 50-digit decimal arithmetic) and NumPy's
expm1 / log2.
"""

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_gemm_b200 import dflash as D

pytestmark = pytest.mark.gpu

SV = O.sampled_verify


def _words():
    rng = np.random.default_rng(5)
    w = rng.integers(0, np.iinfo(np.uint64).max, size=200_000, dtype=np.uint64, endpoint=True)
    ks = [0, 1, 2, (1 << 52) - 1, 1 << 52, 7 * (1 << 50) - 1, 7 * (1 << 50), 7 * (1 << 50) + 1,
          (1 << 53) - 2, (1 << 53) - 1, (1 << 53) - 12345]
    special = np.array(ks, dtype=np.uint64) << np.uint64(11)
    low = np.array([2047] * len(ks), dtype=np.uint64)
    return np.concatenate([w, special, special | low])


def _deltas(n):
    rng = np.random.default_rng(6)
    a = -rng.uniform(0, 40, size=n // 2)
    b = -np.logspace(-30, 1.5, num=n - n // 2)
    edge = [-0.25, np.nextafter(np.float32(-0.25), np.float32(0)),
            np.nextafter(np.float32(-0.25), np.float32(-1)), -1.0, -126.0, -200.0, -1e-30, -np.inf]
    return np.concatenate([a, b, np.array(edge)]).astype(np.float32)


def test_gumbel_and_residual_weight_error_bounds():
    w = _words()
    d = _deltas(len(w))[: len(w)]
    if len(d) < len(w):
        d = np.concatenate([d, -np.ones(len(w) - len(d), dtype=np.float32)])
    wt = torch.from_numpy(w.view(np.int64)).cuda()
    dt = torch.from_numpy(d).cuda()
    g2, l2 = D.debug_sample_math(wt, dt)
    torch.cuda.synchronize()
    g2 = g2.cpu().numpy().astype(np.float64)
    l2 = l2.cpu().numpy().astype(np.float64)

    want_g2 = -np.log2(SV.neg_log_uniform_open(w))
    err_g = np.abs(g2 - want_g2)
    assert np.all(np.isfinite(g2))
    assert err_g.max() <= 2e-5, (err_g.max(), w[np.argmax(err_g)])

    dd = d.astype(np.float64)
    with np.errstate(divide="ignore"):
        want_l2 = np.log2(-np.expm1(dd * np.log(2.0)))
    fin = np.isfinite(dd)
    want_l2[~fin] = 0.0  # d = -inf: 1 - 2^d = 1
    tol = 5e-6 + 3e-7 * np.abs(want_l2)
    err_l = np.abs(l2 - want_l2)
    worst = np.argmax(err_l - tol)
    assert np.all(err_l <= tol), (dd[worst], l2[worst], want_l2[worst])
