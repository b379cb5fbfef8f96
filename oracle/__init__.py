"""CPU oracle of the action-expert denoising loop (test infrastructure only).

Only tests, the smoke check and the bench's CPU-baseline leg may use this package.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import PROJ_INPUTS, E4M3_MAX  # noqa: F401
