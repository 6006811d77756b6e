"""CPU oracle for the ZeroQuant fused quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  The CUDA library never calls
it and it shares no code with the CUDA library.
"""
from .zq_oracle import *  # noqa: F401,F403
