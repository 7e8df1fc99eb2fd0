"""B200-native (sm_100a) GPT-2 causal-LM training step.

The compute path lives in the CUDA shared library ``libgpt.so`` built from
``csrc/``; ``gpt_decoder_lm_b200.binding`` is a thin ctypes binding to its C
ABI (declared in ``include/gpt.h``).  Importing this package does not load
the library; ``binding.lib()`` does, and fails loudly if it is missing.
"""

__all__ = ["binding", "workloads"]
