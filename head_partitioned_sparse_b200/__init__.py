"""Head-partitioned sparse decode attention for B200 (sm_100a).

The CUDA library (``libspa.so``) and its ctypes binding are loaded lazily by
``head_partitioned_sparse_b200.binding``; importing the package itself does not
touch the GPU.  ``synth`` draws seeded synthetic inputs.
"""
__all__ = ["binding", "synth"]
