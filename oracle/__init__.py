"""CPU oracle for the Sign-Muon step (numpy, float64).  TEST INFRASTRUCTURE
ONLY: imported by the tests, the smoke check and the benchmark's CPU-baseline
leg, never by the product path."""
from .signmuon_ref import *  # noqa: F401,F403
from . import signmuon_ref  # noqa: F401
