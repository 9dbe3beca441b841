"""B200-native paged KV-cache decode path (PagedAttention hot path).

The compute lives in ``libpkv.so`` (CUDA kernels for sm_100a plus the host block manager,
behind a C ABI declared in ``include/pkv.h``); ``binding`` marshals torch tensors into that ABI.
Importing this package does not load the library; the first call does, and fails loudly when
the library is missing.
"""
