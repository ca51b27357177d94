"""B200 (sm_100a) HSTU layer forward and M-FALCON scoring behind a C ABI.

The CUDA library (libhstu.so, built by `build.py`) does all the arithmetic;
`hstu` is its ctypes binding.
"""
from . import hstu  # noqa: F401
from .hstu import (HSTUError, Jagged, LayerConfig, LayerWeights, attn_fwd, forward,  # noqa: F401
                   layer_fwd, mfalcon_score)
