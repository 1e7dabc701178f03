"""B200-native grouped linear (ragged grouped GEMM for mixture-of-experts layers).

The compute lives in ``libgl.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/gl.h``); :mod:`grouped_gemm_splits_b200.gl` is the thin
Python binding with the same entry-point names.  Importing this package does
not load the library; the first call into :mod:`.gl` does, and raises if the
library has not been built.
"""
__all__ = ["gl", "synth"]
