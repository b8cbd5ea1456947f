"""B200-native decode-step attention of RTPurbo (head-wise sparse retrieval).

The compute path is the CUDA library ``librtp.so`` behind the C-ABI in ``include/rtp.h``;
``head_wise_sparse_retrieval_b200.rtp`` is its thin ctypes binding. Importing this package
does not load the library; the first call into the binding does, and fails loudly when the
library is missing.
"""
__all__ = ["rtp", "workloads"]
