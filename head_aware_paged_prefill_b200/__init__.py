"""SegPagedAttention prefill for B200 (sm_100a).

The product is the C-ABI library ``librk.so`` built from ``csrc/``; the
Python names below are its thin ctypes binding.  ``synth`` builds seeded
synthetic workloads.
"""
