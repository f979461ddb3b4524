"""STAR-KV latent decode attention for one B200 (sm_100a).

The library is libstarkv.so (C ABI in include/starkv.h); `starkv` is its thin
Python binding.
"""
from . import starkv  # noqa: F401  (fails loudly if libstarkv.so is missing)
from .starkv import Layer, LayerConfig, load_factors, version  # noqa: F401
