"""B200-native MoE layer with zero-computation experts (LongCat-Flash, §2.1).

The compute path is the CUDA library ``libmoe_b200.so`` (sm_100a) behind the
C ABI declared in ``include/moe.h``; ``binding`` marshals torch tensors into
it.  Importing ``configs`` or ``inputs`` needs no GPU.
"""
