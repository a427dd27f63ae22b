"""GPT-2 training step on one NVIDIA B200 (sm_100a): hand-written CUDA kernels
behind a C ABI (include/gpt2.h), with a thin ctypes binding in .gpt2.

Importing the package loads nothing; the CUDA library is loaded on first use
(decoder_only_transformer_02_b200.gpt2.load_library)."""

__all__ = ["gpt2", "synthetic", "build"]
