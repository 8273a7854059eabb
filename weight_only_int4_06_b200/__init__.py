"""libw4a16: group-wise INT4 weight-only quantisation and the W4A16 matmul on B200 (sm_100a).

The compute lives in the CUDA library ``libw4a16.so`` (C ABI declared in ``include/w4a16.h``);
``weight_only_int4_06_b200.w4a16`` is its thin ctypes binding.  ``synth`` holds the seeded
synthetic input generators.
"""
