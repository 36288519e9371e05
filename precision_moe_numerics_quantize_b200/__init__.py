"""nvfp4moe: NVFP4 mixture-of-experts expert layer for B200 (sm_100a).

The compute lives in libnvfp4moe.so (CUDA, built in-tree by build.py); the
``nvfp4moe`` module is its thin ctypes binding and ``synth`` the seeded input
generators. Importing the package does not load the library; the first call
into ``nvfp4moe`` does, and fails loudly if it is missing.
"""
