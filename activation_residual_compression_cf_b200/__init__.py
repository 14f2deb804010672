"""B200-native CompactFusion-style residual compression of exchanged
activations (sender encode with error feedback, receiver decode).

The compute lives in ``libcf.so`` (hand-written sm_100a CUDA kernels behind
the C ABI declared in ``include/cf.h``); ``activation_residual_compression_cf_b200.cf`` is the
thin ctypes binding.  Importing the package loads nothing; the library is
opened on first use and a missing or unbuilt library raises.
"""

__all__ = ["cf", "workloads"]
