"""VideoNSA hybrid sparse-attention layer prefill on B200 (sm_100a).

The compute lives in ``libvnsa.so`` (hand-written CUDA kernels behind a C ABI,
declared in ``include/vnsa.h``); ``binding`` marshals arguments to it through
ctypes.  Importing this package does not load the library; the first call does,
and it raises if the library or a CUDA device is missing -- there is no CPU path.
"""
