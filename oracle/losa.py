"""Oracle: the LoSA sparse variant (locality pruning, page selection, union).

Written from "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
Language Models" (gist.science, es), §2 "El Algoritmo LoSA":
  step 1 (locality pruning): a per-token locality score, the mean squared
    error between this step's and the previous step's query; the tokens with
    the largest change form the active set A, the rest are stable;
  step 2 (cache reuse for stable tokens): stable rows keep the prefix
    statistics (o_p, L_p) stored at the previous step;
  step 3 (sparse attention for active tokens only): a QUEST-like selector
    picks KV subsets I_i for each active query and the KV traffic is the union
    I = U_{i in A} I_i;
  step 4 (merge and update): prefix and block contributions are merged by
    online softmax and the cache takes the new statistics.

The pages name QUEST without defining it. The selector here scores a page of
16 keys by the upper bound sum_c max(q_c * kmin_c, q_c * kmax_c) from per-page,
per-channel key minima and maxima, and keeps the top-k pages per query row and
head.

Decisions (active set, page choice) are integers decided by float scores, so
the scores are computed in a fully specified float32 order that a GPU can
reproduce bit for bit:
  * products and squares are single correctly rounded float32 multiplies;
  * sums use the stride-halving tree: pad to a power of two N with zeros, then
    for stride = N/2, N/4, ..., 1: x[n] <- x[n] + x[n + stride] for n < stride;
    the result is x[0].
  * ties are broken by the lower index.

Test infrastructure only: imported by tests, the smoke check and the bench's
CPU baseline, never by the product path.
"""

from __future__ import annotations

import numpy as np

from .attention import partial, prefix_keys, to_f64


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    return np.asarray(x, dtype=np.float32)


def tree_sum(x: np.ndarray) -> np.ndarray:
    """Stride-halving tree sum over the last axis, in x's own dtype.

    Pad to the next power of two with zeros; then for stride = N/2 ... 1 add
    x[n + stride] into x[n] for n < stride. Every add is one IEEE add of x's
    dtype (numpy does not contract or reorder elementwise adds).
    """
    x = np.asarray(x)
    n = x.shape[-1]
    N = 1
    while N < n:
        N *= 2
    if N != n:
        pad = np.zeros(x.shape[:-1] + (N - n,), dtype=x.dtype)
        x = np.concatenate([x, pad], axis=-1)
    while N > 1:
        N //= 2
        x = x[..., :N] + x[..., N:2 * N]
    return x[..., 0]


# ---------------------------------------------------------------------------
# Step 1: locality score and active set
# ---------------------------------------------------------------------------

def locality_score(q_cur, q_prev, dtype: str) -> np.ndarray:
    """Per block token: sum over all heads and channels of (q_s - q_{s-1})^2.

    q_*: [batch, B, Hq, d]. Returns float32 [batch, B]. The MSE of the pages
    divides this by Hq*d, which changes no ranking and is left out. Order of
    arithmetic: delta = f32(q_cur) - f32(q_prev) (exact for bf16 inputs of
    similar magnitude), delta*delta rounded to float32, tree sum over
    n = h*d + c in float32.
    """
    a = to_f32(q_cur, dtype)
    b = to_f32(q_prev, dtype)
    delta = (a - b).astype(np.float32)
    sq = (delta * delta).astype(np.float32)
    batch, B = sq.shape[:2]
    return tree_sum(sq.reshape(batch, B, -1))


def top_indices(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores (ties: lower index first), in rank order."""
    s = np.asarray(scores, dtype=np.float32)
    n = s.shape[0]
    k = max(0, min(k, n))
    # primary key: score descending (negation is exact); secondary: index
    order = np.lexsort((np.arange(n), -s))
    return order[:k].astype(np.int32)


def active_rows(scores: np.ndarray, n_active: int) -> np.ndarray:
    """Active set per sequence: [batch, min(n_active, B)] rows in rank order."""
    return np.stack([top_indices(scores[b], n_active) for b in range(scores.shape[0])])


# ---------------------------------------------------------------------------
# Step 3: page summaries, page scores, top-k pages, union
# ---------------------------------------------------------------------------

def n_pages(kv, b: int) -> int:
    P = int(kv.page_size)
    return -(-int(kv.seq_len[b]) // P)


def page_summary(kv, dtype: str):
    """Per logical page, kv head and channel: min and max of the page's keys.

    Returns float32 arrays [batch, max_pages, Hkv, d] (exact: min and max of
    bf16 values are bf16 values). Only tokens t < seq_len count, so the last,
    partly filled page is summarised over its valid keys. Pages past a
    sequence's end are NaN.
    """
    batch = len(kv.seq_len)
    P = int(kv.page_size)
    Hkv, d = kv.k.shape[1], kv.k.shape[2]
    maxp = -(-int(kv.max_seq_len) // P)
    smin = np.full((batch, maxp, Hkv, d), np.nan, dtype=np.float32)
    smax = np.full((batch, maxp, Hkv, d), np.nan, dtype=np.float32)
    for b in range(batch):
        n = int(kv.seq_len[b])
        for hk in range(Hkv):
            K, _ = prefix_keys(kv, b, hk, dtype)
            full = n // P  # whole pages, then the ragged last page
            pages = K[: full * P].reshape(full, P, d)
            smin[b, :full, hk] = pages.min(axis=1)
            smax[b, :full, hk] = pages.max(axis=1)
            if full * P < n:
                smin[b, full, hk] = K[full * P: n].min(axis=0)
                smax[b, full, hk] = K[full * P: n].max(axis=0)
    return smin, smax


def page_scores(q_rows: np.ndarray, smin: np.ndarray, smax: np.ndarray) -> np.ndarray:
    """QUEST-style upper bound of q.k over each page.

    q_rows: float32 [R, d]; smin / smax: float32 [n_pages, d].
    u[r, p] = tree_sum_c max(q_c * kmin_{p,c}, q_c * kmax_{p,c}) in float32.
    Returns float32 [R, n_pages].
    """
    q = np.asarray(q_rows, dtype=np.float32)[:, None, :]
    lo = (q * smin[None]).astype(np.float32)
    hi = (q * smax[None]).astype(np.float32)
    return tree_sum(np.maximum(lo, hi))


def select_pages(kv, q, dtype: str, active, topk: int, smin, smax):
    """Top-k pages of every active row and q head, and their union per kv head.

    Returns (chosen, union): chosen[(b, i, h)] = page indices in rank order;
    union[(b, hk)] = sorted page indices chosen by any active row i of sequence
    b and any q head h of kv head hk.
    """
    batch, B, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    qf = to_f32(q, dtype)
    chosen, union = {}, {}
    for b in range(batch):
        npg = n_pages(kv, b)
        for hk in range(Hkv):
            u = set()
            for h in range(hk * G, (hk + 1) * G):
                rows = qf[b, active[b], h]  # [n_active, d]
                if len(active[b]) == 0:
                    continue
                sc = page_scores(rows, smin[b, :npg, hk], smax[b, :npg, hk])
                for r, i in enumerate(active[b]):
                    pick = top_indices(sc[r], topk)
                    chosen[(b, int(i), h)] = pick
                    u.update(int(p) for p in pick)
            union[(b, hk)] = np.asarray(sorted(u), dtype=np.int32)
    return chosen, union


def union_bitmap(union, batch: int, Hkv: int, max_pages: int) -> np.ndarray:
    """Bit p % 32 of word p // 32 set for every page p in the union: uint32."""
    words = -(-max_pages // 32)
    bm = np.zeros((batch, Hkv, words), dtype=np.uint32)
    for (b, hk), pages in union.items():
        for p in pages:
            bm[b, hk, p // 32] |= np.uint32(1 << (p % 32))
    return bm


def sparse_partial(kv, q, dtype: str, active, union, scale: float = 1.0):
    """(o_p, L_p) of the active rows over every key of their kv head's union.

    Returns {(b, i, h): (A [d], L)} for i in active[b].
    """
    batch, B, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    P = int(kv.page_size)
    out = {}
    for b in range(batch):
        if len(active[b]) == 0:
            continue
        n = int(kv.seq_len[b])
        for hk in range(Hkv):
            pages = union[(b, hk)]
            toks = [t for p in pages for t in range(p * P, min(n, (p + 1) * P))]
            K, V = prefix_keys(kv, b, hk, dtype, tokens=np.asarray(toks, dtype=np.int64))
            for h in range(hk * G, (hk + 1) * G):
                rows = to_f64(q[b, active[b], h], dtype)
                A, L = partial(rows, K, V, scale)
                for r, i in enumerate(active[b]):
                    out[(b, int(i), h)] = (A[r], L[r])
    return out
