"""B200-native shifted-window multi-head self-attention over a padded token grid.

The compute lives in ``libswinwattn.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/swin_wattn.h``); ``binding`` marshals torch tensors
into it. Importing this package does not load the library; the first call
does, and fails loudly when it is missing.
"""
from .workloads import WORKLOADS, BENCH_WORKLOAD, Workload  # noqa: F401
