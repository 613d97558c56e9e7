"""certified_top_sparse_b200: certified Top-k attention truncation on B200.

The computation lives in ``libcta.so`` (CUDA, sm_100a), declared in
``include/cta.h``.  This package holds its ctypes binding (``_lib``), the
build script (``build``) and the seeded synthetic workloads (``workloads``).
"""
from ._lib import (  # noqa: F401
    CTA_BF16, CTA_F32, CTA_DEV_INTERNAL, CTA_DEV_NONFINITE, CtaError, EXPORTED, LIB_PATH,
    CTA_ERR_TOO_LARGE, NOALLOC_SCRATCH_BYTES, cta_certified_topk_attn,
    cta_certified_topk_attn_noalloc, cta_dense_attn, cta_status_string, cta_version,
    cta_workspace_size, load,
)
