"""Float64 CPU oracle of the H2O chunk step -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  It shares no code with the CUDA path.
"""
from .h2o_oracle import (H2OHeadOracle, H2OOracle, OracleShapeError, attend_group,
                         select_evictions, select_oldest)
from .brute import brute_stream

__all__ = ["H2OHeadOracle", "H2OOracle", "OracleShapeError", "attend_group",
           "select_evictions", "select_oldest", "brute_stream"]
