"""B200-native RAM-Net layer core: Product-Softmax Top-K address decoding, CAPE, the Gated
Sparse Update and the sparse read with RMSNorm and output gate, as hand-written sm_100a
CUDA kernels behind a C ABI (``include/ramnet.h``).

Importing the package loads nothing; ``sparse_slot_recurrent_b200.ramnet`` loads the
compiled library on first use and raises if it is missing.
"""
__all__ = ["ramnet", "workloads"]
