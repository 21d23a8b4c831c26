"""Seeded synthetic inputs shared by the CPU oracle and the GPU path.

This package holds no arithmetic of the looped nGPT method itself: it only
reads the committed model configs and draws seeded weights, input hidden
states and pre-filled KV-cache contents, so that both implementations can be
fed bit-identical data.  Everything here is plain NumPy, except the optional
torch twin of the KV-cache fill (`kvfill.fill_torch`), which evaluates the same
counter-based hash on the GPU for the multi-GB decode caches.
"""

from .config import load_config, CONFIG_DIR  # noqa: F401
from .bf16 import f32_to_bf16_bits, bf16_bits_to_f32, round_bf16  # noqa: F401
from .weights import block_weights, hidden_in, vocab_weights  # noqa: F401
