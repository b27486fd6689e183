"""B200-native (sm_100a) forward pass of one Mixture-of-Experts layer.

The compute path is the C-ABI library `libmoe.so` (hand-written CUDA kernels);
`expert_router_gemm_b200.moe` is its thin ctypes binding and raises ImportError
when the library has not been built.  `configs` holds the workload shapes and
`synth` the seeded input generator; importing the package loads neither CUDA nor
the library.
"""
from . import configs, synth  # noqa: F401

__all__ = ["configs", "synth"]
