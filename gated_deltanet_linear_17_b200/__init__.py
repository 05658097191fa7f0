"""B200-native (sm_100a) Gated Delta Rule chunked forward.

The compute path is the C-ABI library ``libgdn.so`` (CUDA kernels for
sm_100a); this package only marshals arguments to it.
"""
