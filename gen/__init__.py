"""Seeded synthetic input generation shared by the oracle tests, the GPU tests and the bench."""
from .moe_inputs import *  # noqa: F401,F403
from .moe_inputs import CONFIGS, MoeConfig  # noqa: F401
