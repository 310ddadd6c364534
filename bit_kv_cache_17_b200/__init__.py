"""Mixed-precision KV cache with a BF16 precision tail for NVIDIA B200 (sm_100a).

`kvq` is the thin ctypes binding of libkvq.so (the C ABI declared in include/kvq.h);
`synth` holds the seeded synthetic input generators.  Importing `kvq` loads the CUDA
library and raises if it is missing: there is no CPU fallback.
"""
