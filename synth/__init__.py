"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package generates inputs only: it holds none of the method's arithmetic
(no moments, no shrinkage, no factorisation, no rank or BPW rule).  Both the
CUDA path and the oracle consume what it produces.
"""
from .inputs import *  # noqa: F401,F403
