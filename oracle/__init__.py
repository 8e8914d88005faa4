"""CPU oracle for the BitSSM forward pass: numpy (bitssm_oracle, ssd_oracle),
a plain C host oracle (c/, loaded by c_oracle) held to it, and the
straight-through backward in PyTorch CPU float64 (ste_oracle).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` use it.  It shares no code with the
CUDA library and imports nothing from it.
"""

from .bitssm_oracle import *  # noqa: F401,F403
