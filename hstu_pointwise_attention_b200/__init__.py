"""HSTU pointwise attention on B200 (sm_100a): Python face of libhstu.so.

The compute path is the C-ABI library ``libhstu.so`` (hand-written CUDA for
sm_100a).  ``ops`` only marshals arguments (torch tensors to device pointers
and the params struct) and raises if the library is missing: there is no
fallback path.  ``workloads`` holds the seeded synthetic inputs.
"""
