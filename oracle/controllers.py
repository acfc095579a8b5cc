"""Oracle: the per-step reuse controllers, driven one denoise step at a time.

FlashBlock (gist.science technical summary, §2 "Adaptive reuse strategies"):
  * threshold reuse: with M^{s+1} updated tokens, the cached block-external
    attention is reused when M^{s+1} < tau and recomputed otherwise;
  * per-head selection (video): only heads whose similarity is above gamma
    reuse the cache.
LoSA (gist.science, es, §2 "El Algoritmo LoSA", steps 1-4): stable rows reuse
their cached prefix statistics, active rows get a fresh sparse prefix partial.

Readings where the pages leave a step open:
  * the block is attended bidirectionally (block diffusion is causal between
    blocks only) and the first step of a block has no cache, so it computes;
  * threshold: the decision is per sequence and covers all of its rows and
    heads; M is the count of rows updated since the previous step;
  * per head: a head computes at steps 0 and 1; at a step s >= 1 where it
    computed, c_h = cos(A_out,h^s, A_out,h^{s-1}) over its flattened B x d
    tile; c_h >= gamma makes it reuse for the rest of the block (sticky);
  * the cosine is evaluated in float64 with exact products and the
    stride-halving tree sum, then dot / sqrt(|a|^2 * |b|^2), so that it can be
    replayed bit for bit on the GPU's own float32 tiles.

Test infrastructure only: imported by tests, the smoke check and the bench's
CPU baseline, never by the product path.
"""

from __future__ import annotations

import numpy as np

from . import losa as _losa
from .attention import block_partial, merge, prefix_partial, to_f64


def head_cosine(a: np.ndarray, b: np.ndarray) -> float:
    """Cosine similarity of two tiles in float64 by the specified order.

    a, b: float arrays of equal size (flattened row-major). Products are exact
    in float64 for float32 inputs; sums use the stride-halving tree; the result
    is dot / sqrt(na * nb), or 0 when either tile is all zero.
    """
    x = np.asarray(a, dtype=np.float64).ravel()
    y = np.asarray(b, dtype=np.float64).ravel()
    dot = float(_losa.tree_sum(x * y))
    na = float(_losa.tree_sum(x * x))
    nb = float(_losa.tree_sum(y * y))
    den = na * nb
    if den == 0.0:
        return 0.0
    return dot / float(np.sqrt(den))


class ThresholdController:
    """Threshold (tau) reuse of the block-external partial."""

    def __init__(self, kv, dtype: str, tau: int, scale: float = 1.0):
        self.kv, self.dtype, self.tau, self.scale = kv, dtype, tau, scale
        self.A_out = None
        self.L_out = None

    def step(self, s: int, q, k_in, v_in, m_updated):
        batch = q.shape[0]
        recompute = np.array([s == 0 or int(m_updated[b]) >= self.tau for b in range(batch)])
        if self.A_out is None:
            self.A_out = np.full(q.shape, np.nan)
            self.L_out = np.full(q.shape[:3], np.nan)
        if recompute.any():
            mask = np.repeat(recompute[:, None], q.shape[2], axis=1)
            A, L = prefix_partial(self.kv, q, self.dtype, self.scale, head_mask=mask)
            self.A_out[recompute] = A[recompute]
            self.L_out[recompute] = L[recompute]
        A_in, L_in = block_partial(q, k_in, v_in, self.dtype, self.scale)
        A_full, L_full = merge(self.A_out, self.L_out, A_in, L_in)
        return {"recompute": recompute, "A_full": A_full, "L_full": L_full,
                "A_out": self.A_out.copy(), "L_out": self.L_out.copy()}


class PerHeadController:
    """Per-head (gamma) reuse for video block diffusion.

    ``step(..., a_out_for_decision=...)`` lets a test evaluate the cosine on
    another implementation's A_out tiles (replay), and ``force_mask`` makes this
    controller follow another implementation's decisions (teacher forcing), so
    a float-decided fork cannot separate the two trajectories.
    """

    def __init__(self, kv, dtype: str, gamma: float, scale: float = 1.0):
        self.kv, self.dtype, self.gamma, self.scale = kv, dtype, gamma, scale
        self.A_out = None
        self.L_out = None
        self.mask = None  # [batch, Hq] bool: compute at this step

    def step(self, s: int, q, k_in, v_in, force_mask=None, a_out_for_decision=None):
        batch, B, Hq, d = q.shape
        if self.A_out is None:
            self.A_out = np.full(q.shape, np.nan)
            self.L_out = np.full(q.shape[:3], np.nan)
            self.mask = np.ones((batch, Hq), dtype=bool)
        mask = self.mask.copy() if force_mask is None else np.asarray(force_mask, dtype=bool)
        prev = self.A_out.copy()
        if mask.any():
            A, L = prefix_partial(self.kv, q, self.dtype, self.scale, head_mask=mask)
            sel = np.broadcast_to(mask[:, None, :], (batch, B, Hq))
            self.A_out[sel] = A[sel]
            self.L_out[sel] = L[sel]
        cos = np.full((batch, Hq), np.nan)
        next_mask = mask.copy()
        if s >= 1:
            cur = self.A_out if a_out_for_decision is None else a_out_for_decision[0]
            old = prev if a_out_for_decision is None else a_out_for_decision[1]
            for b in range(batch):
                for h in range(Hq):
                    if mask[b, h]:
                        cos[b, h] = head_cosine(cur[b, :, h, :], old[b, :, h, :])
                        if cos[b, h] >= self.gamma:
                            next_mask[b, h] = False
        self.mask = next_mask
        A_in, L_in = block_partial(q, k_in, v_in, self.dtype, self.scale)
        A_full, L_full = merge(self.A_out, self.L_out, A_in, L_in)
        return {"computed": mask, "cos": cos, "next_mask": next_mask,
                "A_full": A_full, "L_full": L_full,
                "A_out": self.A_out.copy(), "L_out": self.L_out.copy()}


class LosaController:
    """LoSA: dense prefix partial at step 0, sparse refresh of active rows after."""

    def __init__(self, kv, dtype: str, n_active: int, topk: int, scale: float = 1.0):
        self.kv, self.dtype, self.n_active, self.topk, self.scale = kv, dtype, n_active, topk, scale
        self.smin, self.smax = _losa.page_summary(kv, dtype)
        self.A_out = None
        self.L_out = None
        self.q_prev = None

    def step(self, s: int, q, k_in, v_in):
        info = {}
        if s == 0 or self.A_out is None:
            self.A_out, self.L_out = prefix_partial(self.kv, q, self.dtype, self.scale)
        else:
            score = _losa.locality_score(q, self.q_prev, self.dtype)
            act = _losa.active_rows(score, self.n_active)
            chosen, union = _losa.select_pages(self.kv, q, self.dtype, act, self.topk,
                                               self.smin, self.smax)
            fresh = _losa.sparse_partial(self.kv, q, self.dtype, act, union, self.scale)
            for (b, i, h), (a, l) in fresh.items():
                self.A_out[b, i, h] = a
                self.L_out[b, i, h] = l
            info.update(score=score, active=act, chosen=chosen, union=union)
        self.q_prev = np.array(q, copy=True)
        A_in, L_in = block_partial(q, k_in, v_in, self.dtype, self.scale)
        A_full, L_full = merge(self.A_out, self.L_out, A_in, L_in)
        info.update(A_full=A_full, L_full=L_full, A_out=self.A_out.copy(), L_out=self.L_out.copy())
        return info


def dense_step(kv, dtype: str, q, k_in, v_in, scale: float = 1.0):
    """Dense block-diffusion attention, step by step: prefix + block + merge."""
    A_out, L_out = prefix_partial(kv, q, dtype, scale)
    A_in, L_in = block_partial(q, k_in, v_in, dtype, scale)
    return merge(A_out, L_out, A_in, L_in)


__all__ = ["ThresholdController", "PerHeadController", "LosaController",
           "dense_step", "head_cosine", "to_f64"]
