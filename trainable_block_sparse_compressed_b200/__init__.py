"""InfLLM-V2 dense-sparse switchable attention for NVIDIA B200 (sm_100a).

The compute lives in ``libinfllmv2.so`` (CUDA kernels behind a C ABI, see
``include/infllmv2.h``); :mod:`.infllmv2` is the thin ctypes binding with the
same entry-point names.  :mod:`.workloads` generates seeded synthetic inputs.
"""
