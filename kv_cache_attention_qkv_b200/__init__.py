"""B200-native Flash-Cache step: QKV projection + RoPE + KV-cache write,
bidirectional variable-length attention with per-key importance, and top-k
reselection of the tracked positions, behind the C-ABI library
``libflashcache.so`` (declared in ``include/flashcache.h``).

``FlashCache`` (in :mod:`.binding`) is the Python face of that library; it only
marshals arguments.  Importing it loads the CUDA library and raises if the
library has not been built: there is no fallback.
"""
import importlib

__all__ = ["FlashCache", "FlashCacheModel", "FlashCacheError", "load_library"]


def __getattr__(name):
    if name in __all__:
        return getattr(importlib.import_module(__name__ + ".binding"), name)
    raise AttributeError(name)
