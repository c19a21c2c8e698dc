"""B200-native paged-attention decode: KV append into fixed-size blocks,
single-query decode attention gathered through a block table, and
copy-on-write block copies, behind a small C-ABI library of sm_100a kernels.

Importing the package loads nothing; the CUDA library is loaded by the
binding on first use and a missing library is an error, never a fallback.
"""
