"""B200-native hybrid-head sparse decode attention (LycheeDecode's decode step).

The compute path is the C-ABI library ``liblyc.so`` (hand-written sm_100a CUDA
kernels); ``hybrid_head_sparse_b200.lyc`` is its thin ctypes binding.  Import
that module to use the library; it raises if the library is not built.
"""
