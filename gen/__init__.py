"""Seeded synthetic inputs (shapes, value distributions, storage formats) for the routed-expert layer."""
from .configs import CONFIGS, MoEConfig, get  # noqa: F401
from . import inputs  # noqa: F401
