"""B200-native DSA decode step: lightning-indexer scan, top-k, sparse MQA.

The compute lives in the CUDA library ``liblsa.so`` (C ABI, include/lsa.h);
``lsa`` is its thin ctypes binding.  ``synth`` builds seeded synthetic inputs.
"""
__all__ = ["lsa", "synth"]
