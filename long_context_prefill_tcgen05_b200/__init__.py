"""B200-native Delta-Attention Selective Halting (DASH) long-context prefill.

The compute path is the C-ABI library ``libdash.so`` (hand-written CUDA for
sm_100a, declared in ``include/dash.h``); ``dash`` is its thin ctypes binding.
Importing this package does not load the library; ``dash.lib()`` does, and
raises if it is missing.
"""
