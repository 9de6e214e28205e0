"""B200-native (sm_100a) separator-sparse attention and SepCache streaming decode.

The compute lives in libsepattn.so (CUDA kernels behind a C ABI, see include/sepattn.h);
`kv_cache_compression_sep_b200.sepattn` is its ctypes binding. Import that module to use the
library; it raises if the library has not been built.
"""

__all__ = ["sepattn"]
