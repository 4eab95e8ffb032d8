"""B200-native microscaling (MXFP8 / MXFP4 / NVFP4) quantize + block-scaled GEMM.

The compute path is the C-ABI library ``libmx.so`` built from ``csrc/`` for
sm_100a; ``mx`` is its thin ctypes binding (argument marshalling only).
"""
