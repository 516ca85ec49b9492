"""B200-native paged KV-cache decode path (sm_100a CUDA behind a C-ABI library).

``synth`` builds seeded synthetic workloads. The device entry points are bound
in ``_binding`` (loaded on first use; it raises if the CUDA library is missing).
"""
