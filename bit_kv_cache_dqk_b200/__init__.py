"""libdualqk: B200 (sm_100a) decode hot path of Dual-QK -- paired key/query
transforms, INT2 KV cache with BF16 key channel 0, query-channel-pruned
split-K attention over a paged cache.

``dualqk`` is the ctypes binding of the C ABI (include/dualqk.h); ``inputs``
draws seeded synthetic workloads; ``build`` compiles the CUDA library.
"""
