"""NVFP4 W4A4 linear layer for Blackwell (sm_100a).

The compute path is the CUDA library ``libmq.so`` (kernels in ``csrc/``, C ABI
declared in ``include/mq.h``); :mod:`.mq` is its thin ctypes binding and
:mod:`.inputs` holds the seeded synthetic workloads.
"""
