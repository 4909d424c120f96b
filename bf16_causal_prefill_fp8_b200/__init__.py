"""B200-native causal prefill attention with the ZYFA FP8 method.

The compute path is the CUDA library libzyfa.so (csrc/, C-ABI declared in
include/zyfa.h); `zyfa` is its thin ctypes binding and `synth` draws seeded
synthetic inputs.
"""
