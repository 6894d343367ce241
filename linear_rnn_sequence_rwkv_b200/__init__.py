"""B200-native (sm_100a) WKV-7 recurrence of RWKV-7 "Goose".

The compute lives in the CUDA library ``lib/libwkv7.so`` behind the C ABI of
``include/wkv7.h``; ``wkv7`` is its thin ctypes binding. ``inputs`` draws the
seeded synthetic workloads. Importing this package does not load the library;
``wkv7.load()`` does, and raises if it has not been built.
"""
__all__ = ["wkv7", "inputs", "build"]
