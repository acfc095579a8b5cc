"""Block commit: the finished block joins the block-external cache.

TEST INFRASTRUCTURE (see oracle/__init__.py). Block diffusion generates
block-wise causally (FlashBlock abstract; technical summary §2): once a block
is final, its keys and values become part of J_out for every later block, and
the LoSA selector's per-page key summaries (LoSA §2 step 3) must then cover
the new tokens too. This module states that update plainly: copy the block's
rows into the cache slots of positions n .. n+B-1 of each sequence and extend
seq_len. The summaries of the grown cache are simply oracle.losa.page_summary
of it, recomputed from scratch.
"""

from __future__ import annotations

import dataclasses

import numpy as np


def block_commit(prefix, k_in: np.ndarray, v_in: np.ndarray):
    """A new prefix equal to `prefix` with block rows k_in/v_in [batch, B, Hkv, d]
    appended to every sequence (token n_b + j <- block row j).

    Slot of token t (the cache's own addressing):
      paged:      page_table[b, t // P] * P + t % P
      contiguous: b * max_seq_len + t
    Raises ValueError when a sequence would outgrow max_seq_len or, paged, the
    pages its table maps.
    """
    batch, B = k_in.shape[0], k_in.shape[1]
    P = int(prefix.page_size)
    k = prefix.k.copy()
    v = prefix.v.copy()
    seq_len = prefix.seq_len.copy()
    for b in range(batch):
        n = int(seq_len[b])
        if n + B > int(prefix.max_seq_len):
            raise ValueError(f"sequence {b}: {n} + {B} tokens exceed max_seq_len")
        for j in range(B):
            t = n + j
            if prefix.page_table is None:
                slot = b * int(prefix.max_seq_len) + t
            else:
                page = int(prefix.page_table[b, t // P])
                if page < 0:
                    raise ValueError(f"sequence {b}: logical page {t // P} is not mapped")
                slot = page * P + t % P
            k[slot] = k_in[b, j]
            v[slot] = v_in[b, j]
        seq_len[b] = n + B
    return dataclasses.replace(prefix, k=k, v=v, seq_len=seq_len)
