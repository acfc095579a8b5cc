"""Oracle: packed (variable-length) block rows.

BlockBatch page (gist.science, es), "Optimización del Sistema": the unmasked
query positions of all active branches are packed into one variable-length
buffer, so that branches with different block sizes run in one forward. A
branch is a sequence of the batch here, with its own block of B_b rows and its
own block-external keys (J_out through the cache). Packing changes the layout
only: sequence b owns packed rows cu[b] .. cu[b+1]-1, and every quantity of the
FlashBlock decomposition (technical summary, §2 "Core mechanism") is the
per-sequence one. The oracle therefore runs the per-sequence definitions of
attention.py over each packed segment in turn, with no blocking beyond that.

Test infrastructure only (tests, the smoke check, the bench's CPU baseline).
"""

from __future__ import annotations

import numpy as np

from .attention import merge, partial, prefix_keys, to_f64


def segments(cu):
    """(b, r0, r1) of every sequence: its rows are r0 .. r1-1 of the packed buffers."""
    cu = [int(x) for x in cu]
    return [(b, cu[b], cu[b + 1]) for b in range(len(cu) - 1)]


def prefix_partial_varlen(kv, q, cu, dtype: str, scale: float = 1.0):
    """(A_out, L_out) of every packed row over its own sequence's prefix keys.

    q: [total, Hq, d] storage array; q head h reads kv head h // (Hq / Hkv).
    Returns A [total, Hq, d], L [total, Hq] (float64).
    """
    total, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    A = np.full((total, Hq, d), np.nan)
    L = np.full((total, Hq), np.nan)
    for b, r0, r1 in segments(cu):
        if r1 == r0:
            continue
        for hk in range(Hkv):
            K, V = prefix_keys(kv, b, hk, dtype)
            for h in range(hk * G, (hk + 1) * G):
                a, l = partial(to_f64(q[r0:r1, h], dtype), K, V, scale)
                A[r0:r1, h], L[r0:r1, h] = a, l
    return A, L


def block_partial_varlen(q, k_in, v_in, cu, dtype: str, scale: float = 1.0):
    """(A_in, L_in): every row of sequence b against the B_b keys of its own
    block (rows r0 .. r1-1 of k_in / v_in), bidirectional."""
    total, Hq, d = q.shape
    Hkv = k_in.shape[1]
    G = Hq // Hkv
    A = np.full((total, Hq, d), np.nan)
    L = np.full((total, Hq), np.nan)
    for b, r0, r1 in segments(cu):
        if r1 == r0:
            continue
        for h in range(Hq):
            a, l = partial(to_f64(q[r0:r1, h], dtype), to_f64(k_in[r0:r1, h // G], dtype),
                           to_f64(v_in[r0:r1, h // G], dtype), scale)
            A[r0:r1, h], L[r0:r1, h] = a, l
    return A, L


class ThresholdVarlenController:
    """Threshold (tau) reuse over packed rows: sequence b recomputes its
    block-external partial at step 0 or when m_updated[b] >= tau (FlashBlock,
    "Adaptive reuse strategies"); every step the block partial is recomputed
    and merged with the cached one."""

    def __init__(self, kv, dtype: str, tau: int, scale: float = 1.0):
        self.kv, self.dtype, self.tau, self.scale = kv, dtype, tau, scale
        self.A_out = self.L_out = None

    def step(self, s: int, q, k_in, v_in, cu, m_updated):
        segs = segments(cu)
        recompute = np.array([s == 0 or self.tau <= 0 or int(m_updated[b]) >= self.tau
                              for b, _, _ in segs])
        if self.A_out is None:
            self.A_out = np.full(q.shape, np.nan)
            self.L_out = np.full(q.shape[:2], np.nan)
        if recompute.any():
            A_new, L_new = prefix_partial_varlen(self.kv, q, cu, self.dtype, self.scale)
        for (b, r0, r1), rec in zip(segs, recompute):
            if rec:
                self.A_out[r0:r1], self.L_out[r0:r1] = A_new[r0:r1], L_new[r0:r1]
        A_in, L_in = block_partial_varlen(q, k_in, v_in, cu, self.dtype, self.scale)
        A_full, L_full = merge(self.A_out, self.L_out, A_in, L_in)
        return {"recompute": recompute, "A_full": A_full, "L_full": L_full}
