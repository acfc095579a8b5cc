"""Oracle for per-denoise-step block-diffusion attention (FlashBlock, LoSA).

TEST INFRASTRUCTURE. A plain, slow, float64 CPU statement of what the GPU
path computes, written from the FlashBlock and LoSA pages and pinned by tests
against closed forms, brute force and invariants. Only tests/, the smoke check
in __graft_entry__ and the bench's CPU baseline may import it; the product
package never does, and it shares no code with the CUDA path.

Modules:
  attention    partials over a key set, the log-space merge, dense attention
  losa         locality score, active set, page summaries and scores, top-k
               pages, union, sparse partial
  controllers  threshold (tau), per-head (gamma) and LoSA step procedures
  cache        block commit: a finished block's K/V appended to the cache
  residual     FlashBlock + sparse attention: cached residual of unselected pages
  varlen       packed (variable-length) block rows of several sequences
"""

from . import attention, cache, controllers, losa, residual, varlen  # noqa: F401
from .attention import (  # noqa: F401
    block_partial,
    dense_attention,
    merge,
    partial,
    prefix_partial,
    prefix_partial_samples,
    to_f64,
)
