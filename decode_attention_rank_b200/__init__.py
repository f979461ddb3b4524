"""STAR-KV latent decode attention for one B200 (sm_100a).

The library is libstarkv.so (C ABI in include/starkv.h); `starkv` is its thin
Python binding.  Importing `decode_attention_rank_b200.starkv` (or any name
below) fails loudly if libstarkv.so is missing: there is no fallback path.
The binding is loaded on first use so that `python -m
decode_attention_rank_b200.build` can run before the library exists.
"""
import importlib

_EXPORTS = ("Layer", "LayerConfig", "load_factors", "version", "StarKVError")


def __getattr__(name):
    if name == "starkv" or name in _EXPORTS:
        mod = importlib.import_module(__name__ + ".starkv")
        return mod if name == "starkv" else getattr(mod, name)
    raise AttributeError(name)
