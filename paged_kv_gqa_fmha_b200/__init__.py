"""B200 (sm_100a) paged-KV grouped-query attention engine.

The attention runs in ``libpa_b200.so`` (hand-written CUDA kernels behind the C
ABI of ``include/pa.h``); ``binding.Plan`` is its Python binding.  Build the
library with ``python -m paged_kv_gqa_fmha_b200._build``.
"""
from .binding import Plan, PAError, load_library  # noqa: F401
