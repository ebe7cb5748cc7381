"""B200-native hot path of Latent Sparse Attention with a hierarchical latent-key index.

The compute runs in the CUDA library ``liblsa.so`` (C ABI declared in
``include/lsa.h``); :mod:`hierarchical_latent_key_b200.lsa` is its thin binding.
"""
