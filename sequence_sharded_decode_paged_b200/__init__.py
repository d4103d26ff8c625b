"""B200-native decode context parallelism: sharded paged-KV decode attention.

The compute path is the CUDA library ``libdcp.so`` (C ABI in
``include/dcp.h``); ``sequence_sharded_decode_paged_b200.dcp`` is its thin
ctypes binding.  Import the binding explicitly::

    from sequence_sharded_decode_paged_b200 import dcp

It raises ImportError when the library has not been built.
"""
__all__ = ["dcp"]
