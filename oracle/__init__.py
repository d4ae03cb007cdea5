"""fp64 CPU oracle of the hybrid-block attention path -- test infrastructure only.

Imported only by tests/, the build entry point's smoke check and the
benchmark's CPU-baseline leg. The product library never imports it.
"""
from .hs_oracle import *  # noqa: F401,F403
from .hs_oracle import make_tiles, Tile  # noqa: F401
