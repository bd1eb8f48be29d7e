"""B200-native exact attention: FlashAttention-style prefill and paged decode on sm_100a.

The compute path is the C-ABI library ``libattn_b200.so`` (hand-written CUDA for sm_100a);
``exact_attention_161_b200.api`` is its thin Python binding (argument marshalling only).
Importing this package loads nothing; ``api`` loads the library on import and raises if it
is missing -- there is no CPU fallback.
"""

__all__ = ["api", "synth"]


def __getattr__(name):
    if name in ("api", "synth"):
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
