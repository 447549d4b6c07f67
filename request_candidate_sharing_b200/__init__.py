"""librocs: the ROCS (Request-Oriented Compute Sharing) forward hot path on NVIDIA B200.

The compute lives in librocs.so (CUDA for sm_100a, C ABI in include/rocs.h); `rocs` is its
ctypes binding and `build` compiles it in-tree.  Importing `request_candidate_sharing_b200.rocs`
raises if the library has not been built.
"""
