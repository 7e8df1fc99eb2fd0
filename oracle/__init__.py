"""CPU oracle for the GPT-2 causal-LM training step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow, float64 restatement of the step that the nanoGPT /
microGPT pages describe, written with numpy; ``numpy.matmul`` (a BLAS call)
is the only library primitive it leans on.  It shares no code, tables or
constants with the CUDA library in ``gpt_decoder_lm_b200/``.
"""

from .gpt_oracle import *  # noqa: F401,F403
