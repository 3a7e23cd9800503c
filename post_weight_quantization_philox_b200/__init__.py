"""GSQ Gumbel-Softmax layer-reconstruction step on NVIDIA B200 (sm_100a).

The compute lives in ``libgsq.so`` (hand-written CUDA behind the C ABI of
``include/gsq.h``); :mod:`.gsq` is its thin ctypes binding and :mod:`.synth`
draws the seeded synthetic workloads.
"""
__all__ = ["gsq", "synth", "build"]
