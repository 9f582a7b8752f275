"""SageAttention-style quantized attention forward pass for NVIDIA B200 (sm_100a).

``sageattn(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None,
smooth_k=True)`` smooths K (and optionally Q, V), quantises Q/K to INT8 and V
to FP8 e4m3, and runs a tcgen05/TMEM/TMA attention kernel (INT8 Q K^T, FP8
P V).  The compute lives in ``libsage_b200.so`` (C ABI: include/sage_b200.h);
this package only marshals arguments.
"""
from .binding import SageError, sageattn, sageattn_varlen  # noqa: F401

__all__ = ["sageattn", "sageattn_varlen", "SageError"]
