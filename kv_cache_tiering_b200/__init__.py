"""B200-native tiered KV-history decode attention.

The compute path is the C-ABI CUDA library ``libakv`` (``csrc/``, declared in
``include/akv.h``); ``kv_cache_tiering_b200.akv`` is its thin ctypes binding and
``kv_cache_tiering_b200.synth`` generates seeded synthetic inputs.  Neither is imported
here, so the input generator can be used without the built library.
"""
