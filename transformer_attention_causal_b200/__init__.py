"""B200-native causal (MHA / GQA / MQA) scaled-dot-product attention.

The compute lives in ``libb200attn.so`` (CUDA C++ for sm_100a behind a C ABI,
declared in ``include/b200attn.h``); this package is a thin binding to it.
"""
