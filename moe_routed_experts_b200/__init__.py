"""B200-native frozen AWQ routed-experts MoE FFN.

The compute path is the C-ABI library ``libmoe_awq.so`` (hand-written CUDA for
sm_100a, declared in ``include/moe_awq.h``); ``binding`` marshals PyTorch
device tensors into it.  ``inputs`` and ``configs`` describe the synthetic
workloads.  Importing the package does not load the library; the first call
through ``binding`` does, and fails loudly if it is missing.
"""
