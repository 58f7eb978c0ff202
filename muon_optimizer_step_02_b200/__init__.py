"""Fused batched Muon optimizer step and batched EMA for NVIDIA B200.

The compute path is the C-ABI library ``libmuonb200.so`` (hand-written
sm_100a CUDA); :mod:`.binding` is a thin ctypes layer over it and loads it on
first use.  :mod:`.workloads` holds the seeded synthetic inputs.
"""

__all__ = ["binding", "workloads"]
