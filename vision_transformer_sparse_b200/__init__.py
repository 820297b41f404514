"""B200-native Bi-Level Routing Attention (BRA) forward.

The compute path is the C-ABI library `libbra.so` built from `csrc/` (CUDA for
sm_100a); `bra.py` is its thin ctypes binding. `synth.py` draws the seeded
synthetic inputs used by the tests and the benchmark.
"""
