"""B200 (sm_100a) implementation of the Ideogram 4 DiT block forward.

The C-ABI library (``libig4.so``, built from ``csrc/`` by ``build.py``) holds
every kernel; ``stream_diffusion_transformer_fwd_b200.ig4`` is its Python
binding and fails to import if the library is missing.
"""
