"""Multipole Attention decode for NVIDIA B200 (sm_100a).

Clustered sparse decode attention ("Multipole Attention for Efficient Long
Context Reasoning"): keys are grouped by blockwise k-means; each decode step
attends exactly to the top clusters up to a token budget and approximates the
rest by count-weighted centroid terms.  The work runs in the CUDA library
libmpattn.so (C ABI in include/mpattn.h); this package is its Python binding.
"""
from .api import Config, MultipoleIndex, dense_decode, workspace_size  # noqa: F401
from ._lib import MpError  # noqa: F401
