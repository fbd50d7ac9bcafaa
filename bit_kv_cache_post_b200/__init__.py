"""WUSH-KV low-bit KV cache on B200: Python binding of libwushkv.so.

``wushkv`` marshals arguments to the C ABI declared in include/wushkv.h;
``inputs`` draws the seeded synthetic workloads.  Importing the package does
not load the CUDA library; the first call that needs it does, and fails
loudly if it has not been built.
"""
