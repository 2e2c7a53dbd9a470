"""Routed mixture-of-experts FFN layer for B200 (sm_100a).

The compute path lives in ``libmoe.so`` (CUDA kernels behind a C ABI, declared
in ``include/moe.h``).  ``routed_expert_ffn_forward_b200.moe`` is the thin ctypes
binding with the same names; ``synth`` draws seeded synthetic inputs.
"""
