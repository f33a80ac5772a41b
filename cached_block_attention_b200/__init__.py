"""cached_block_attention_b200: cached block attention for block-diffusion decoding on B200.

``fbk`` (the CUDA library binding) is loaded on first access so that ``synth``
(seeded inputs) can be imported on hosts without the built library.
"""
import importlib

__all__ = ["fbk", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
