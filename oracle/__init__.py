"""CPU oracle for the NVFP4 MoE expert-layer path. TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never calls it.
"""
from .oracle import *  # noqa: F401,F403
