"""Packed (variable-length) block rows: several branches of different block
sizes in one launch, shaped after the BlockBatch page ("Optimización del
Sistema": the unmasked query positions of all active branches in one
variable-length buffer; the page's branches use block sizes such as 4, 8, 16,
32, 64 and 128 for the same request).

Layout only: a batched workload is drawn with the largest block size, and
sequence b keeps the first rows[b] rows of its block. With shared_prefix, every
branch reads the same prefix pages through its page table (branches of one
request share the request's KV cache); this needs a paged base workload.
No attention arithmetic lives here.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Iterator, Optional, Sequence

import numpy as np

from .gen import Prefix, make_workload

BLOCKBATCH_ROWS = (4, 8, 16, 32, 64, 128)


@dataclass
class VarlenStep:
    step: int
    q: np.ndarray  # [total, Hq, d]
    k_in: np.ndarray  # [total, Hkv, d]
    v_in: np.ndarray
    m_updated: np.ndarray  # int32 [batch]


class VarlenWorkload:
    def __init__(self, base: str, rows: Sequence[int], shared_prefix: bool = False, **ov):
        self.rows = [int(r) for r in rows]
        batch = len(self.rows)
        self.base = make_workload(base, batch=batch, block=max(max(self.rows), 1), **ov)
        self.spec = self.base.spec
        self.cu = np.concatenate([[0], np.cumsum(self.rows)]).astype(np.int32)
        self.total = int(self.cu[-1])
        pre = self.base.prefix
        if shared_prefix:
            if pre.page_table is None:
                raise ValueError("shared_prefix needs a paged base workload")
            n = int(pre.seq_len[0])
            used = -(-n // pre.page_size)
            table = np.repeat(pre.page_table[:1], batch, axis=0)
            table[:, used:] = -1
            pre = Prefix(pre.k, pre.v, np.full(batch, n, dtype=np.int32), table, pre.page_size,
                         pre.max_seq_len)
        self.prefix = pre

    def steps(self, n_steps: Optional[int] = None) -> Iterator[VarlenStep]:
        for st in self.base.steps(n_steps):
            yield VarlenStep(
                st.step,
                np.concatenate([st.q[b, :r] for b, r in enumerate(self.rows)]),
                np.concatenate([st.k_in[b, :r] for b, r in enumerate(self.rows)]),
                np.concatenate([st.v_in[b, :r] for b, r in enumerate(self.rows)]),
                np.minimum(st.m_updated, np.asarray(self.rows, dtype=np.int32)).astype(np.int32))


def make_varlen_workload(base: str, rows: Sequence[int] = BLOCKBATCH_ROWS,
                         shared_prefix: bool = False, **ov) -> VarlenWorkload:
    return VarlenWorkload(base, rows, shared_prefix, **ov)
