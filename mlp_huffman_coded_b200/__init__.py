"""Lossless Huffman-coded BF16 MLP weights with a reconstructive GEMM on B200.

The compute lives in the C-ABI library ``libuw.so`` (hand-written sm_100a
CUDA plus a C++ host codec); ``mlp_huffman_coded_b200.uw`` is its thin ctypes
binding.  Importing this package does not load the library: ``uw.lib()``
does, and fails loudly when the library has not been built.
"""

__all__ = ["uw", "synth"]
