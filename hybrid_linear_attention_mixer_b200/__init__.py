"""B200-native Gated DeltaNet token mixer.

``hybrid_linear_attention_mixer_b200.gdn`` is the Python binding of the C-ABI
library (``libgdn_b200.so``); importing this package does not load it.
"""
__all__ = ["gdn", "inputs"]
