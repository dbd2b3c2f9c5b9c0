"""Online INT8 W8A8 linear and routed-MoE kernels for B200 (sm_100a).

The compute lives in the C-ABI library ``libw8a8.so`` (``csrc/``); the
Python module :mod:`moe_gemm_absmax_b200.w8a8` is a thin ctypes binding
with the same entry-point names.  There is no CPU fallback: calling an
entry point without the built library raises.
"""
__all__ = ["w8a8", "inputs"]
