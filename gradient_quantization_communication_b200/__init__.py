"""B200-native bucketed gradient quantization for communication.

The hot path (error feedback, per-bucket level fit, Philox stochastic rounding, dense bit
packing, decode and worker average) runs in the CUDA library ``libgq.so`` behind the C ABI in
``include/gq.h``; ``gq`` is its Python binding and ``synth`` draws seeded synthetic gradients.
"""
from . import gq  # noqa: F401
