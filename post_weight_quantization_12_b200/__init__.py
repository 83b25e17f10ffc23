"""GPTQ layer quantization for NVIDIA B200 (sm_100a).

The compute lives in libgptq_b200.so (hand-written CUDA, C ABI in include/gptq.h); this package
holds the ctypes binding (`_lib`), a convenience layer that allocates buffers with PyTorch and
calls the three entry points (`api`), the in-tree build script (`build`) and seeded synthetic
inputs (`synth`).
"""
__all__ = ["api", "synth"]
