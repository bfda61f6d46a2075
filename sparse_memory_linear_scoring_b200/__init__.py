"""Sparse Delta Memory (SDM) forward pass on NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in include/sdm.h (libsdm.so, built in-tree by
`python -m sparse_memory_linear_scoring_b200.build`).  Every step of the pass
runs in the library's CUDA kernels; this package only marshals torch tensors
into pointers and the current CUDA stream.  There is no CPU path: calling
without the built library, or with CPU tensors, raises.
"""
from .sdm import (  # noqa: F401
    SDMError, Dims, LIB_PATH, load_library, workspace_bytes, forward, forward_decay, step, select,
    recur, backward,
    device_status, make_dims, query_plan, PLAN_FIELDS, gdn_forward, gdn_workspace_bytes, GdnDims,
)
