"""fp64 CPU oracle of the VMoBA layer -- test infrastructure only.

Importable only from the tests, the smoke check and the bench's CPU-baseline
leg; the CUDA library shares no code with it.
"""
from .vmoba_oracle import *  # noqa: F401,F403
