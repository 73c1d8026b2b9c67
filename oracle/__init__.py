"""CPU oracle for the padding-free MoE layer -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the layer computes, written from the
X-MoE descriptions and shared with nothing in ``padding_free_moe_b200``.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import it; the product path never does.
"""
from .moe_oracle import *  # noqa: F401,F403
