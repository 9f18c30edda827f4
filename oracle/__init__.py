"""CPU oracle of the ASR audio-encoder forward pass (test infrastructure).

This package is the correctness reference for the CUDA library and nothing
else: only the tests, the smoke check and the benchmark's CPU-baseline leg
import it.  The product path never calls it, and it shares no code with the
CUDA library (the two meet only at the seeded input generators in ``synth``).

Everything is float64 numpy, written as the plain definition of each step,
with library primitives (matrix multiply, erf) used as steps and no blocking
or fusion beyond what the definition states.  Each function cites the passage
of the pages it follows.  The pages are three web pages; they are cited by
title and section:

  [MOSS]   "MOSS-Transcribe-preview-2B-GGUF" model card (Architecture table,
           Implementation notes table, Non-obvious gotchas).
  [CW]     "CrisperWhisper -> ONNX (with cross-attentions)" (What this exports
           instead; Results).

Parity status of every function is listed in ``oracle.forward``'s module
docstring.
"""
from .forward import *  # noqa: F401,F403
