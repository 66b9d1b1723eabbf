"""B200-native HSTU jagged pointwise attention and transduction layer.

The compute path is the C-ABI library `libhstu.so` (CUDA, sm_100a); the
Python binding in `hstu_sequential_transduction_b200.ops` only marshals
arguments.  `workloads` draws seeded synthetic inputs and `flops` holds the
algorithmic FLOP / byte accounting.
"""

__all__ = ["workloads", "flops"]
