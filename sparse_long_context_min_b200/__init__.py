"""EntmaxKV support-aware paged decoding for alpha-entmax attention on B200 (sm_100a).

One decode step over a paged KV cache: score pages from their metadata
(bounding boxes, Gaussian moments), select candidate pages (top-k or the
Gaussian-aware tau_hat rule), and run exact alpha-entmax attention over the
gathered pages -- all in the CUDA library behind include/entmaxkv.h.  This
package is the thin Python binding (``binding``), the in-tree build
(``build``), the decode-step driver (``step``) and the seeded synthetic
workloads (``workloads``).
"""
from . import binding  # noqa: F401
from .binding import (  # noqa: F401
    Pool, EntmaxKVError, append_metadata, score_pages, select, sparse_attend, full_entmax_decode,
    full_softmax_decode, workspace_size, status_string, selftest_timeout,
)
