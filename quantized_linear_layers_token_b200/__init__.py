"""B200-native outlier-aware W4A8 / W8A8 quantized linear layer.

The compute lives in ``libqlin.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/qlin.h``); :mod:`.qlin` is a thin ctypes binding with
the same entry-point names.
"""
