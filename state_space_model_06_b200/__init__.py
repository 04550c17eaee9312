"""Mamba-3 SSM mixer hot path for B200 (sm_100a).

``m3`` is the thin binding of the C ABI in ``include/m3.h`` (libm3.so, built
in-tree by ``build.py``); ``inputs`` draws the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .m3 import *  # noqa: F401,F403
