"""B200-native (sm_100a) fused GQA attention forward and split-KV decode.

The compute lives in ``libgqa_attn.so`` (hand-written CUDA, C ABI declared in
``include/gqa_attn.h``); ``gqa_attention_flash_b200.binding`` is the thin
ctypes layer over it.  ``gqa_attention_flash_b200.workloads`` draws the seeded
synthetic inputs.  Importing this package loads neither.
"""
__all__ = ["binding", "workloads"]
