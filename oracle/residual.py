"""FlashBlock combined with sparse attention: cached residual of the unselected keys.

TEST INFRASTRUCTURE (see oracle/__init__.py). FlashBlock technical summary
§2, "Compatibility with sparse attention": FlashBlock is orthogonal to sparse
attention; it treats the keys a sparse method does not select as the
"block-external" set and caches their residual contribution, which recovers
the information that aggressive sparsification drops.

Readings taken here, where the pages name the idea but no procedure:
  * the sparse selector is the QUEST-style page bound the LoSA page uses
    (§2 step 3), applied per kv head: head score of page p =
    max over block rows i and the G q heads h of that kv head of
    u[i, h, p] = tree_sum_c max(q_c kmin_{p,c}, q_c kmax_{p,c}) (float32, the
    specified order); the top-k pages (ties: lower page) form the selected
    set S, every other page of the sequence the complement C;
  * refresh (new selection and new residual) follows the threshold rule:
    step 0, tau <= 0, or any sequence with M >= tau (a batched step shares one
    selection pass, so all sequences refresh together);
  * at a refresh the residual (A_C, L_C) = partial over C with the current q is
    stored; every step computes the fresh sparse partial (A_S, L_S) over S with
    the current q and A_out = merge(A_S, L_S, A_C, L_C); then the in-block
    partial is merged as in FlashBlock.
Consequences used as pins: at a refresh S and C split J_out exactly, so A_out
equals the dense prefix partial; top-k >= pages gives C empty (dense every
step); top-k = 0 gives S empty (plain FlashBlock threshold reuse).
"""

from __future__ import annotations

import numpy as np

from . import losa as _losa
from .attention import block_partial, merge, partial, prefix_keys, to_f64


def head_page_scores(kv, q, dtype: str, b: int, hk: int, smin, smax) -> np.ndarray:
    """float32 [n_pages]: max over rows and the kv head's q heads of the page bound."""
    Hq = q.shape[2]
    G = Hq // kv.k.shape[1]
    npg = _losa.n_pages(kv, b)
    qf = _losa.to_f32(q, dtype)
    rows = qf[b][:, hk * G:(hk + 1) * G, :].reshape(-1, qf.shape[-1])  # r = i * G + g
    u = _losa.page_scores(rows, smin[b, :npg, hk], smax[b, :npg, hk])
    return u.max(axis=0)


def head_selection(kv, q, dtype: str, topk: int, smin, smax):
    """{(b, hk): (S, C)}: selected and complementary pages, ascending."""
    batch = q.shape[0]
    Hkv = kv.k.shape[1]
    out = {}
    for b in range(batch):
        npg = _losa.n_pages(kv, b)
        for hk in range(Hkv):
            sc = head_page_scores(kv, q, dtype, b, hk, smin, smax)
            sel = np.sort(_losa.top_indices(sc, topk)).astype(np.int32)
            comp = np.setdiff1d(np.arange(npg, dtype=np.int32), sel)
            out[(b, hk)] = (sel, comp)
    return out


def pages_partial(kv, q, dtype: str, pages, scale: float = 1.0):
    """(A, L) [batch, B, Hq, d] / [batch, B, Hq]: every row over the tokens of
    its kv head's pages (pages[(b, hk)]). An empty page set gives A = 0, L = -inf."""
    batch, B, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    P = int(kv.page_size)
    A = np.zeros((batch, B, Hq, d))
    L = np.full((batch, B, Hq), -np.inf)
    for b in range(batch):
        n = int(kv.seq_len[b])
        for hk in range(Hkv):
            toks = [t for p in pages[(b, hk)] for t in range(p * P, min(n, (p + 1) * P))]
            K, V = prefix_keys(kv, b, hk, dtype, tokens=np.asarray(toks, dtype=np.int64))
            for h in range(hk * G, (hk + 1) * G):
                a, l = partial(to_f64(q[b, :, h], dtype), K, V, scale)
                A[b, :, h] = a
                L[b, :, h] = l
    return A, L


class SparseResidualController:
    """Sparse attention over selected pages plus FlashBlock's cached residual."""

    def __init__(self, kv, dtype: str, tau: int, topk: int, scale: float = 1.0):
        self.kv, self.dtype, self.tau, self.topk, self.scale = kv, dtype, tau, topk, scale
        self.smin, self.smax = _losa.page_summary(kv, dtype)
        self.sel = None
        self.A_res = self.L_res = None

    def step(self, s: int, q, k_in, v_in, m_updated):
        batch = q.shape[0]
        refresh = (s == 0 or self.sel is None or self.tau <= 0 or
                   any(int(m_updated[b]) >= self.tau for b in range(batch)))
        if refresh:
            self.sel = head_selection(self.kv, q, self.dtype, self.topk, self.smin, self.smax)
            comp = {key: c for key, (_, c) in self.sel.items()}
            self.A_res, self.L_res = pages_partial(self.kv, q, self.dtype, comp, self.scale)
        selected = {key: sp for key, (sp, _) in self.sel.items()}
        A_s, L_s = pages_partial(self.kv, q, self.dtype, selected, self.scale)
        A_out, L_out = merge(A_s, L_s, self.A_res, self.L_res)
        A_in, L_in = block_partial(q, k_in, v_in, self.dtype, self.scale)
        A_full, L_full = merge(A_out, L_out, A_in, L_in)
        return {"refresh": refresh, "selection": self.sel, "A_out": A_out, "L_out": L_out,
                "A_full": A_full, "L_full": L_full}
