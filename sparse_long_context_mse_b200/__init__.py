"""LoSA per-denoising-step attention for B200 (sm_100a).

The compute lives in the CUDA library ``liblosa.so`` behind the C ABI of
``include/losa.h``; :mod:`.api` is its thin Python binding and
:mod:`.synth` draws the seeded synthetic workloads.
"""
__all__ = ["api", "synth"]
