"""B200-native (sm_100a) Q4_0 decode/encode hot path of Voxtral Mini 4B Realtime.

The kernels and their C ABI live in ``libvox.so`` (sources under ``csrc/``,
declarations in ``include/vox.h``); :mod:`.vox` is the thin ctypes binding and
:mod:`.workloads` builds the synthetic decoder / encoder state on the GPU.
Importing the package does not load the library; importing ``.vox`` does, and
fails loudly if it has not been built.
"""
__all__ = ["vox", "workloads", "build"]
