"""CPU oracle of the block-wise diffusion denoise step (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference arms may import this package; the CUDA library never does.
"""
from . import twotower_oracle  # noqa: F401
