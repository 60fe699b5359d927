"""B200-native MLA absorbed decode over a paged latent KV cache.

The compute lives in the CUDA shared library built from ``csrc/`` (see
``mla_latent_kv_29_b200.lib``); this package only marshals arguments.
Importing the package does not load the library: the first call does, and it
raises ``RuntimeError`` if the library is missing or no GPU is visible.
"""
