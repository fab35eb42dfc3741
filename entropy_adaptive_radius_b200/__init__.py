"""Token Radius Attention hot path for B200 (sm_100a).

The compute path is the C-ABI library libtra.so (hand-written CUDA kernels);
`entropy_adaptive_radius_b200.tra` is its thin ctypes binding.  Importing the
package does not load the library; the binding loads it on first use and
raises if it is missing.
"""
__all__ = ["tra", "inputs", "workloads"]
