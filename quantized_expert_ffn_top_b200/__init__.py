"""B200-native routed MoE expert FFN layer (NVFP4 / MXFP4 / FP8 W8A8).

The compute path lives in the C-ABI library ``libmoe_b200.so`` built from
``csrc/`` (sm_100a CUDA).  ``ops`` is the thin ctypes binding; it loads the
library on first use and raises if it is missing -- there is no CPU fallback.
``synth`` draws the seeded synthetic inputs.
"""
__all__ = ["ops", "synth"]
