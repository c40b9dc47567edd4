"""CPU oracle of the displaced-patch UNet layer step (numpy, fp64).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the benchmark's CPU-baseline leg, never by the product path.
"""
from .dfp_oracle import *  # noqa: F401,F403
