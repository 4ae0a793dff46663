"""fp8_moe_numerics_b200 -- B200-native (sm_100a) numerics of 4-bit MoE training.

NVFP4 quantisation of activations and expert weights, grouped NVFP4 expert
GEMMs on tcgen05 block-scaled tensor cores, the dequantise -> transpose ->
stochastic-rounding MXFP8 requantisation of saved tensors, and the MXFP8
dgrad/wgrad grouped GEMMs, behind the C ABI in include/mxmoe.h.

The CUDA library (libmxmoe.so) is loaded on first use; importing this package
does not touch the GPU.
"""
from .api import *  # noqa: F401,F403
from .api import max_routed_rows  # noqa: F401
