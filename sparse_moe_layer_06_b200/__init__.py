"""B200 (sm_100a) sparse Mixture-of-Experts FFN layer forward.

The compute lives in the CUDA library ``libmoe_b200.so`` (C ABI in
``include/moe.h``); :mod:`sparse_moe_layer_06_b200.moe` is its thin Python
binding and :mod:`sparse_moe_layer_06_b200.workloads` draws the seeded inputs.
Importing the package does not load the library; the first call does, and it
fails loudly if the library has not been built.
"""
from .workloads import CONFIGS, MoEConfig, make_inputs  # noqa: F401
