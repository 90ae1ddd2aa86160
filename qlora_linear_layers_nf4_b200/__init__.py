"""B200-native NF4 quantization and QLoRA linear layers.

The compute lives in a C-ABI shared library (libnf4qlora.so, CUDA for
sm_100a) declared in include/nf4qlora.h; `nf4qlora` is its thin ctypes
binding.  PyTorch is used only for device memory and streams.
"""
__all__ = ["nf4qlora", "workloads"]
