"""Loki-style low-rank-key sparse decode attention for NVIDIA B200 (sm_100a).

The compute lives in libloki.so (CUDA C++, C ABI declared in include/loki.h);
`rank_key_top_b200.loki` is the thin ctypes binding with the same names.
"""
