"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This package only *describes and fills* inputs: context lengths, block tables,
slot mappings, copy-on-write pairs and bf16 tensors drawn from N(0, 1).  It holds
none of the attention arithmetic, and it imports neither the oracle nor the CUDA
library.
"""
from .synth import *  # noqa: F401,F403
