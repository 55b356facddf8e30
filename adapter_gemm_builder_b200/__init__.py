"""Multi-tenant LoRA apply on B200 (sm_100a).

The compute path is the C-ABI library ``liblora.so`` (CUDA kernels for
sm_100a, declared in ``include/lora.h``); :mod:`adapter_gemm_builder_b200.lora`
is its thin ctypes binding. :mod:`adapter_gemm_builder_b200.workloads` draws
the seeded synthetic inputs.
"""
