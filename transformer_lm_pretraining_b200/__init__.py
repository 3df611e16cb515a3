"""B200-native GPT-2 pretraining step.

The step (forward, backward, global-norm clip, AdamW) runs in hand-written
sm_100a CUDA kernels behind a C ABI (``include/gpt2.h``); ``gpt2`` is the
ctypes binding.  Importing the package loads nothing: the binding loads the
CUDA library on first use and raises if it is missing.
"""
