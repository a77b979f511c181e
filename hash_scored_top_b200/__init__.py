"""hash_scored_top_b200: hash-scored top-k sparse decode attention on B200.

The compute path is the C-ABI library ``libhash_scored_top.so`` (CUDA kernels
for sm_100a); the Python functions here only marshal torch tensors into it.
"""
