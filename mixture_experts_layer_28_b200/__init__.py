"""B200-native MoE layer with zero-computation experts (LongCat-Flash style).

The compute path is the C-ABI library ``libmoe_zc.so`` (hand-written CUDA for
sm_100a); :mod:`.moe_zc` is its thin ctypes binding and loads it on first
use.  :mod:`.workloads` holds the seeded synthetic inputs.
"""
__all__ = ["moe_zc", "workloads"]
