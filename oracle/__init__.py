"""CPU oracle of the routed-expert layer (float64 numpy).

Test infrastructure only: the tests, the smoke check and the benchmark's CPU
baseline may import it; the CUDA product path never does.
"""
from . import moe_oracle  # noqa: F401
