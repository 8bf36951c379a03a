"""Oracle for EntmaxKV support-aware paged decoding.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
CPU restatement of what one EntmaxKV decode step computes, in float64 unless a
function says otherwise.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  The CUDA library never calls
it, shares no code with it and has no fallback to it.

Sources (the EntmaxKV pages: the German and Hindi technical summaries of
"EntmaxKV: Support-Aware Decoding for Entmax Attention" and the paper's
abstract):

* ``entmax``  -- alpha-entmax itself (section 2: exact zeros for alpha > 1);
  the definition p_i = [x_i - tau]_+^{1/(alpha-1)}, sum p = 1.
* ``pages``   -- per-page metadata and the bounding-box bound (section 2.A:
  coordinatewise k_min/k_max, first and second moments).
* ``gauss``   -- the Gaussian-aware threshold estimate tau_hat (section 2.B,
  policy 2: an approximate normalisation equation from page statistics).
* ``select``  -- top-k and Gaussian keep rules (section 2.B).
* ``attend``  -- exact entmax attention over kept tokens, full-cache entmax
  and softmax baselines, dropped mass delta (sections 2.C, 3, 4).
* ``replica`` -- fp32 canonical-order replicas of the quantities whose
  floating-point value decides an integer (which pages are selected): the
  page metadata, the bound and the Gaussian page estimates.  These are taken
  in fp32 in a fixed operation order so that both sides decide in the same
  precision.

Parity pins that are NOT fixed by the pages (they print no formula for tau_hat
and no estimator for a page's maximum): the Gaussian normalisation equation
(``gauss.F``) and the page-maximum estimate (``gauss.z_table``) follow this
build's reading; they are pinned to closed forms, Monte-Carlo and quadrature,
but whether they equal the paper's own selector is parity unpinned.
"""

from . import entmax, pages, gauss, select, attend, replica  # noqa: F401
