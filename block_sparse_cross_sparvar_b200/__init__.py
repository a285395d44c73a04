"""B200-native SparVAR block-sparse cross-scale attention.

The compute path is the C-ABI library ``libsparvar.so`` (hand-written sm_100a
CUDA kernels); ``ops`` binds its entry points under the same names.
"""
