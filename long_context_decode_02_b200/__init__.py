"""LowRAM decode hot path on B200: C-ABI library ``liblowram.so`` plus a thin binding.

``long_context_decode_02_b200.lowram`` loads the compiled library (and raises if it is
missing); ``long_context_decode_02_b200.synth`` makes seeded synthetic workloads.
Importing the package itself loads nothing.
"""
