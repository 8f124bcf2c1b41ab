"""CPU oracle for the grouped NVFP4 MoE expert forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import anything from here.
The product path (the CUDA library and its Python binding) never does.
"""

from .nvfp4_moe_oracle import *  # noqa: F401,F403
