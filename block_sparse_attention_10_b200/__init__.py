"""B200-native MiniMax-Sparse-Attention (MSA) decode over an NVFP4 KV cache.

The compute path is hand-written CUDA for sm_100a in ``libmsa.so`` behind a C
ABI (``include/msa.h``); :mod:`.msa` is its thin ctypes binding (argument
marshalling only).  :mod:`.synth` and :mod:`.configs` describe the synthetic
workloads.
"""
