"""CPU oracles of the Sparse Delta Memory forward pass and of the dense Gated
DeltaNet baseline -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports or calls it; it shares no code with it.
"""
from .oracle import (  # noqa: F401
    build, compile_source, load, forward, forward_decay, select, forward_head, ORACLE_SO,
    ORACLE_SRC,
    load_gdn, gdn_forward, GDN_SO, GDN_SRC,
)
