"""TileShare shared transformer layer for B200 (sm_100a).

The compute path lives in the C-ABI library ``libtileshare.so`` (hand-written CUDA
for sm_100a); ``binding`` is a thin ctypes layer over it.  The library is loaded on
first use and a missing library raises; there is no fallback.
"""
