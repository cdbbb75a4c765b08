"""fp64 CPU oracle for the MLA latent-KV hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library does
not use it, and it does not use the CUDA library: the two share no code.
"""

from .mla_oracle import *  # noqa: F401,F403
