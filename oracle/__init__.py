"""fp64 CPU oracle of the SSA hot path.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are its only callers.  The product path never
imports it, and it imports nothing from the product package.
"""
from .ssa_oracle import *  # noqa: F401,F403
