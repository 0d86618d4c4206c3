"""B200-native DFlash block-diffusion speculative-decoding hot path.

The work happens in ``libdflash.so`` (CUDA kernels for sm_100a behind the C
ABI in include/dflash.h); ``dflash`` is its ctypes binding.  Build the library
with ``python -m block_diffusion_speculative_gemm_b200.build``.
"""

from . import dflash  # noqa: F401
from .dflash import (  # noqa: F401
    DFlashError,
    Model,
    draft_block,
    get_error,
    inject_kv,
    new_workspace,
    timing_enable,
    timing_read,
    verify,
    verify_workspace_size,
)
