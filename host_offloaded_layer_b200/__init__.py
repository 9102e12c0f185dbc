"""B200 layer-streaming training hot path (MegaTrain-style) behind a C ABI.

The product is ``libmt.so`` (sources in ``csrc/``, declarations in
``include/mt.h``); ``_lib`` is its ctypes binding, ``synth`` the seeded
synthetic inputs and ``metrics`` the throughput formulas. Importing the
package does not load the library; ``_lib.load()`` does, and fails loudly
when it has not been built.
"""
