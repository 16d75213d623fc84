"""ctypes front end of the fp64 CPU oracle (dflash_oracle.c), plus the
temperature-sampling rule and its counter-based random numbers (sampling.py).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg.  The product package never imports it, and this
module imports nothing from the product package.
"""
from .build import build_oracle, oracle_lib_path
from .api import OracleSpec, OracleSession, load_lib

__all__ = ["build_oracle", "oracle_lib_path", "OracleSpec", "OracleSession", "load_lib"]
