"""FlashHead two-stage classification head for B200 (sm_100a).

Submodules:
  flashhead  — ctypes binding of the CUDA library libflashhead.so (the product path)
  synth      — seeded synthetic indices and queries
  costmodel  — algorithmic bytes/flops of a head call (the roofline numerators)
  _build     — nvcc build of the CUDA library

Importing the package loads nothing; ``flashhead`` loads the CUDA library on first use and raises
if it is missing.
"""

__all__ = ["flashhead", "synth", "costmodel"]
