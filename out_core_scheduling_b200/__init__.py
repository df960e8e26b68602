"""B200-native CQS-decomposed exact attention (Stream-CQSA forward path).

The compute lives in the C-ABI library ``libcqsa.so`` (CUDA for sm_100a plus
a C++ planner and streaming scheduler); ``cqsa`` is its thin ctypes binding.
Importing this package does not load the library; the first call does.
"""
