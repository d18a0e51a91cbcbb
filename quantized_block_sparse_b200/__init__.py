"""B200-native SageSLA attention (INT8 SageAttention x Sparse-Linear Attention).

The compute path is the CUDA library ``libsagesla.so`` (C ABI, see include/sagesla.h);
``quantized_block_sparse_b200.sagesla`` is a thin ctypes binding over it. Importing this
package does not load the library; the first call does, and fails loudly if it is missing.
"""
__all__ = ["inputs", "sagesla"]
