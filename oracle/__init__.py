"""fp64 CPU oracle of the Fast-dLLM v2 block-diffusion decoding step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may call it.  It shares no code with
the CUDA library and imports nothing from ``decoding_bd_block_b200``; the two
meet only through the seeded inputs of ``decoding_bd_block_b200.workloads``.

Every function here is written plainly, in float64, following the passage of
the method notes it cites; see ``bd_oracle`` for the list and the readings
taken where the pages leave a step open.
"""
from .bd_oracle import *  # noqa: F401,F403
