"""The bounds-checked build (libdflash_checked.so, compiled with DFLASH_CHECKED):
index checks at the addressing points that depend on device data (the
attention's TMA row of every key tile, the K/V destination of every injected
row, the compact LM-head rows of the commit) set DFLASH_DEV_CHECK and skip the
access instead of trapping.  The small parity tests run once against it in a
child process; every one of them asserts a clean device error word, so a
failed check fails them.  This stands in for a memory checker, which is not
available on the GPUs these tests run on."""

import os
import subprocess
import sys

import pytest

from block_diffusion_speculative_gemm_b200 import build as Bld

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_under_the_bounds_checked_build():
    lib = Bld.build(checked=True)
    env = dict(os.environ, DFLASH_LIB=lib)
    env.pop("DFLASH_PARITY_RECORD", None)
    sel = ("tests/test_draft_gpu.py::test_draft_tiny tests/test_draft_gpu.py::test_draft_small_8b_geometry "
           "tests/test_draft_gpu.py::test_draft_context_lengths_edge_cases "
           "tests/test_draft_gpu.py::test_draft_attention_chunk_sizes "
           "tests/test_inject_gpu.py::test_inject_tiny_prefill "
           "tests/test_inject_gpu.py::test_inject_small_batched_steady_and_prefill "
           "tests/test_paged_kv_gpu.py::test_paged_injection_and_draft_match_contiguous_and_oracle "
           "tests/test_paged_kv_gpu.py::test_paged_prefix_sharing "
           "tests/test_verify_gpu.py tests/test_graph_gpu.py").split()
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        *sel], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
