"""B200-native (sm_100a) RetNet retention operator.

The compute lives in libret.so (C ABI, include/ret.h); `ret` is its thin
binding. Importing the package does not load the library: call
``linear_attention_ret_b200.ret.load()`` (the binding's functions do it).
"""
__all__ = ["ret", "inputs", "build"]
