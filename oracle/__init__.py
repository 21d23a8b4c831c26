"""CPU oracle for the looped nGPT (Dory) forward pass.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import or run
anything in this package.  The product path (the CUDA library and its Python
binding) never imports it and fails loudly when its extension is missing.

The oracle is a plain, slow, obviously-correct NumPy implementation in float64
(weights and inputs are the bf16 values of the shared synthetic generators,
held exactly in float64).  It shares no code with the GPU path.  `quant`
holds the block-scaled weight formats of the quantised checkpoints (MXFP8,
NVFP4): codecs, block quantisation, dequantisation.
"""

from .ngpt_oracle import (  # noqa: F401
    Oracle, KVCache, l2norm, rope, is_full_layer, block_role, kv_cache_bytes,
    layer_applications, weights_from_generator, mask_allows,
)
