"""Longformer banded + global self-attention for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``liblf.so`` built from ``csrc/``; the
module :mod:`sparse_attention_banded_b200.lf` is its thin ctypes binding.
Importing the package does not load the library.
"""
