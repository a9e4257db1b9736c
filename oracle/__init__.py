"""Plain float64 CPU oracle of the CLHA calibration path.

TEST INFRASTRUCTURE. Only the tests, the package smoke check and the bench's CPU-baseline /
reference legs may import it. The product path (the CUDA library and its Python binding) never
calls it and has no CPU fallback.
"""
from .clha_oracle import *  # noqa: F401,F403
