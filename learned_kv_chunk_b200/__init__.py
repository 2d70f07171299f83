"""B200 (sm_100a) implementation of the FlashMemory DS-V4 retriever hot path.

The compute lives in libfm.so (C ABI, include/fm.h); `learned_kv_chunk_b200.fm`
is its ctypes binding.  Importing the binding loads the library and raises if
it has not been built (`python -m learned_kv_chunk_b200.build`).
"""
