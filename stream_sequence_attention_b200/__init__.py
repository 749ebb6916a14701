"""B200-native Hidden Decoding hot path: n-table expansion, Stream-Factorized
Attention (intra / cross, GQA, window), per-stream KV-cache decode and the
final-stream gather, each backed by a hand-written sm_100a CUDA kernel behind
a C ABI (``include/hd.h``).  ``hd`` holds the ctypes binding."""

__version__ = "0.1.0"
