"""fp64 CPU oracle of the wave-index method (test infrastructure only).

Only tests/, the package smoke check and the bench's CPU-baseline leg import
this package.  See wave_oracle.py for the definitions and their sources.
"""
from .wave_oracle import *  # noqa: F401,F403
