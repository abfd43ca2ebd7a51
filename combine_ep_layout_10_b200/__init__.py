"""B200-native (sm_100a) MoE expert-parallel layout / dispatch / combine.

The compute path is the CUDA library libep_b200.so (C ABI in include/ep.h);
`combine_ep_layout_10_b200.ep` is its Python binding and
`combine_ep_layout_10_b200.group.EpGroup` runs the same contract across GPUs
(one process each).  Importing the package does not load the library; the
first call does, and raises if it is missing.
"""
from .ep import (EpError, Handle, LayoutResult, ep_combine, ep_dispatch, ep_handle_free,
                 ep_layout, ep_max_recv_rows)

__all__ = ["EpError", "Handle", "LayoutResult", "ep_combine", "ep_dispatch", "ep_handle_free",
           "ep_layout", "ep_max_recv_rows"]
