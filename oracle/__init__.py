"""Test infrastructure: the plain fp64 CPU oracle (see relpos_oracle.py).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import it.
"""
from .relpos_oracle import *  # noqa: F401,F403
from .relpos_oracle import RelCfg, backward, backward_rows, default_scale, forward, index_map, t5_bucket, table_rows  # noqa: F401
