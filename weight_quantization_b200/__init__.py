"""B200-native TQ3 KV codec and OrbitQuant RPBH weight path.

The compute lives in the CUDA library ``libwq_b200.so`` (C ABI declared in ``include/wq.h``);
``weight_quantization_b200.ops`` is the thin Python binding over it. Importing the package does
not load the library; the first call does, and fails loudly if it is missing.
"""
__all__ = ["inputs", "ops"]
