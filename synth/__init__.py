"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's
callers.  Holds no arithmetic of the MoE method (see ``synth.gen``)."""
from .gen import *  # noqa: F401,F403
