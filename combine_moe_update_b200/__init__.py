"""B200-native MoE token update-expert / dispatch / combine+Add+RMSNorm.

The compute runs in hand-written sm_100a CUDA kernels behind a C ABI
(``include/moe_b200.h``); ``combine_moe_update_b200.binding`` is the thin
ctypes layer over it.  ``combine_moe_update_b200.inputs`` draws the seeded
synthetic workloads.  Submodules are imported lazily so that the input
generators can be used without loading the CUDA library.
"""
__all__ = ["binding", "inputs"]
