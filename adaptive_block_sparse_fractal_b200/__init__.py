"""B200-native NABLA block-sparse 3D attention.

The compute path is the C-ABI library ``libnabla.so`` (CUDA kernels for
sm_100a) declared in ``include/nabla.h``; ``nabla`` is its thin ctypes
binding.  Importing this package does not load the library: ``nabla.lib()``
does, and it raises if the library was not built.
"""
__all__ = ["nabla", "synth"]
