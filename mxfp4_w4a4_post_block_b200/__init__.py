"""libbatq: B200-native BATQuant W4A4 MXFP4 linear path.

The compute lives in the C-ABI shared library ``libbatq.so`` (hand-written
CUDA for sm_100a).  ``mxfp4_w4a4_post_block_b200.batq`` is the thin ctypes
binding with the same call names; ``workloads`` holds the seeded synthetic
input generators.  The library is loaded on first use and the binding raises
if it is missing: there is no CPU fallback.
"""
