"""B200-native deterministic MoE layer (forward + backward) behind a C ABI.

The compute runs in ``libmoe.so`` (hand-written sm_100a kernels); this package
only marshals arguments (``binding``) and draws seeded inputs (``inputs``).
The shared library is loaded on first use, not at import.
"""
