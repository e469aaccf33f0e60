"""HARD-KV decode step on B200 (sm_100a): C-ABI library + thin Python binding.

Importing the package loads nothing; ``attention_kv_head_b200.lib()`` loads the
compiled ``libhardkv.so`` and fails loudly if it is missing.
"""

__all__ = ["lib"]


def lib():
    from . import binding
    return binding.load()
