"""CPU oracle for the Multi-Router Latent MoE layer: the forward pass
(mrlmoe_oracle), its backward (mrlmoe_backward) and its expert-parallel form
(mrlmoe_ep).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its binding) never calls it, and it shares no code with
the CUDA path: its only common dependency is the seeded input generator in
``workloads``.
"""
from .mrlmoe_oracle import *  # noqa: F401,F403
