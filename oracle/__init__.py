"""CPU oracle of the two-stage DDIM denoiser.

TEST INFRASTRUCTURE: imported only by tests/, the smoke check and the
benchmark's CPU-baseline leg.  The library never imports it.
"""
from .kimodo_oracle import *  # noqa: F401,F403
from .kimodo_oracle import Shape, param_count, unpack_weights  # noqa: F401
