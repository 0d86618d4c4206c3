"""fp64 CPU oracle for the DFlash draft hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
library and its Python binding never call it, and it shares no code with them.
"""

from .dflash_oracle import *  # noqa: F401,F403
from .dflash_oracle import __all__  # noqa: F401
from . import sampled_verify  # noqa: F401
from . import sampled_draft  # noqa: F401
from . import paged_kv  # noqa: F401
from . import vocab_parallel  # noqa: F401
