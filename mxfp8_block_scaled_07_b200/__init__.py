"""B200-native MXFP8 quantize / scale-swizzle / block-scaled GEMM / grid-equality library.

The compute lives in ``libmx.so`` (hand-written CUDA for sm_100a behind a C ABI, declared in
``include/mx.h``). ``mxfp8_block_scaled_07_b200.mx`` is the thin ctypes binding; importing
this package does not load the shared library, so the seeded input generators in
``synth`` stay usable on hosts without a GPU.
"""
