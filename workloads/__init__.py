"""Seeded synthetic workloads: the generators (synth) and the five layer configurations (configs)."""
from . import synth, configs  # noqa: F401
