"""B200-native (sm_100a) forward pass of the looped normalized-GPT stack.

The compute path is the C-ABI shared library `libdory.so` (include/dory.h):
tcgen05/TMEM GEMMs with fused epilogues, FlashAttention-style prefill and
split-KV decode attention, nGPT row updates, and a CUDA-graph loop
controller.  `binding` is the ctypes layer; `model` holds the torch buffers.
"""

from . import binding  # noqa: F401
