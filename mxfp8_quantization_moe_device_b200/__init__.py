"""B200-native dynamic FP8 / MXFP8 quantization for MoE training.

The compute lives in the sm_100a CUDA library ``libmxq.so`` (C ABI declared in
``include/mxq.h``); ``binding`` marshals torch tensors into it.
"""
