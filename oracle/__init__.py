"""Float64 CPU oracle for head-wise sparse decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
imports nothing from the CUDA library or its binding, and the library never
imports it.
"""

from .sparse_decode_oracle import *  # noqa: F401,F403
from .head_classifier_oracle import *  # noqa: F401,F403
from .prefill_oracle import *  # noqa: F401,F403
