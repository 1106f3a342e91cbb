"""B200-native DeepSeek-Sparse-Attention lightning indexer (dense, MISA, HISA).

The compute path is a C-ABI shared library of hand-written sm_100a CUDA
kernels (``csrc/``, built in-tree as ``libdsa_indexer.so``). ``binding``
marshals torch device tensors into that ABI; ``workloads`` builds seeded
synthetic inputs.
"""
