"""fp64 CPU oracle of the MoE-layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check of `__graft_entry__` and the CPU-baseline leg
of `bench.py` may import this package.  The library path never calls it and
shares no code with it; the only common module is `workload`, which draws the
seeded inputs.
"""
from .moe_oracle import *  # noqa: F401,F403
from .fp8 import *  # noqa: F401,F403
