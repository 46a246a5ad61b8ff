"""GPT-OSS MXFP4 mixture-of-experts feed-forward layer for NVIDIA B200 (sm_100a).

The layer runs entirely in the hand-written CUDA kernels of ``libmoe_b200.so``
behind the C ABI of ``include/moe.h``; ``mxfp4_expert_ffn_bias_b200.moe`` is the
ctypes binding. Importing the binding raises if the library is missing: there
is no fallback implementation.
"""

import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")
