"""B200-native masked-diffusion LLM block-decode step (KV cache + threshold commit).

The compute path is the C-ABI CUDA library ``libdllm.so`` built from ``csrc/``;
``abi`` is its thin ctypes binding.  Importing this package does not load the
library; the first use of ``abi`` does, and fails loudly if it is missing.
"""
__all__ = ["workload"]
