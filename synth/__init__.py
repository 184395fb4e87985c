"""Seeded synthetic workload generators (no method arithmetic)."""
from .inputs import *  # noqa: F401,F403
