"""B200-native DoSA certified indexer Top-K: a C-ABI CUDA library (libdosa)
with a thin ctypes binding.  The binding only marshals arguments; every step of
the indexer runs in the library's sm_100a kernels."""
