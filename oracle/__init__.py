"""CPU oracle for the routed-expert MoE layer -- TEST INFRASTRUCTURE ONLY.

Imported only by tests, the smoke check and the benchmark's CPU-baseline
leg.  It shares no code with the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
from .gap import enforce_logit_gap  # noqa: F401
from . import mx  # noqa: F401
