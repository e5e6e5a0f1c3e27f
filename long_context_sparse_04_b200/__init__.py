"""B200-native DeepSeek Sparse Attention forward path (indexer, top-k, sparse MLA).

Importing the package does not load the CUDA library; ``native()`` does.
"""
__all__ = ["native"]


def native():
    from . import _native
    return _native
