"""Float64 CPU oracle for attention forward/backward.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the library itself.
"""
from .ref import *  # noqa: F401,F403
from .ref import __all__  # noqa: F401
