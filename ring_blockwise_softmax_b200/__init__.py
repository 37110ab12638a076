"""B200-native blockwise / ring softmax attention (forward).

The compute path is a C-ABI shared library of hand-written sm_100a CUDA kernels
(``csrc/``, declared in ``include/ra_attn.h``).  ``ring_blockwise_softmax_b200.ra_attn``
is the thin ctypes binding; importing it loads the library and raises if the
library has not been built.  ``inputs`` holds the seeded workload generators.
"""
