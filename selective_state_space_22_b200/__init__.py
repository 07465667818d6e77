"""B200-native chunked selective state-space (SSD) scan.

The compute lives in ``libssd.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/ssd.h``); this package only marshals arguments.
"""
