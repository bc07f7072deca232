"""B200-native tree-verify MLA attention (absorbed form).

The compute path is the C-ABI library ``libkdv.so`` (hand-written CUDA for
sm_100a, declared in ``include/kdv.h``); ``kdv`` is its thin Python binding.
Importing this package does not load the library; ``kdv.load()`` does, and
raises if the library is missing.
"""
__all__ = ["datagen", "kdv"]
