"""Oracle: block-external / block-internal attention partials and their merge.

Plain fp64 numpy, written from the FlashBlock pages:
  "FlashBlock: Attention Caching for Efficient Long-Context Block Diffusion",
  technical summary (gist.science, pt and ja), §2 Methodology, "Core mechanism":
  the attention over all keys J is split into keys inside the current block
  (J_in) and outside it (J_out); each part yields an output A and a log
  normaliser L = log Z, and the two are combined by the log-space composition
      A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}),
      m = max(L_out, L_in).

Test infrastructure only: imported by tests, the smoke check and the bench's
CPU baseline, never by the product path.
"""

from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array (float32, or uint16 bf16 bits) -> float64, exactly."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


def partial(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float = 1.0):
    """Softmax attention of query rows over one key set, with its log normaliser.

    q: [R, d], K, V: [N, d] (float64). Scores s_rj = scale * <q_r, k_j>.
    Returns A [R, d] = sum_j softmax_j(s_r) v_j and L [R] = log sum_j e^{s_rj}
    (natural log). Two passes: the row maximum first, then the exponentials
    shifted by it, so nothing overflows. An empty key set gives A = 0 and
    L = -inf (the neutral element of the merge).
    """
    q = np.asarray(q, dtype=np.float64)
    R, d = q.shape
    if K.shape[0] == 0:
        return np.zeros((R, V.shape[1] if V.ndim == 2 else d)), np.full(R, -np.inf)
    s = scale * (q @ K.T)  # [R, N]
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    Z = e.sum(axis=1)
    A = (e @ V) / Z[:, None]
    L = m + np.log(Z)
    return A, L


def merge(A_out, L_out, A_in, L_in):
    """The FlashBlock log-space composition of two partials.

    A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m})
    with m = max(L_out, L_in), and the merged normaliser
    L_full = m + log(e^{L_out-m} + e^{L_in-m}) (not printed on the pages; it is
    the log of Z_out + Z_in, which is what a further merge needs).
    Shapes: A [..., d], L [...]. A side with L = -inf contributes nothing; if
    both are -inf the result is A = 0, L = -inf.
    """
    A_out = np.asarray(A_out, dtype=np.float64)
    A_in = np.asarray(A_in, dtype=np.float64)
    L_out = np.asarray(L_out, dtype=np.float64)
    L_in = np.asarray(L_in, dtype=np.float64)
    m = np.maximum(L_out, L_in)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w_out = np.where(empty, 0.0, np.exp(L_out - m_safe))
    w_in = np.where(empty, 0.0, np.exp(L_in - m_safe))
    den = w_out + w_in
    den_safe = np.where(empty, 1.0, den)
    A = (w_out[..., None] * A_out + w_in[..., None] * A_in) / den_safe[..., None]
    L = np.where(empty, -np.inf, m_safe + np.log(den_safe))
    return A, L


# ---------------------------------------------------------------------------
# Key sets of a workload
# ---------------------------------------------------------------------------

def token_slots(kv, b: int) -> np.ndarray:
    """Pool slot of every prefix token of sequence b, in token order.

    Paged pool: token t is slot page_table[b, t // P] * P + t % P.
    Contiguous pool (no page table): token t is slot b * max_seq_len + t.
    """
    n = int(kv.seq_len[b])
    t = np.arange(n, dtype=np.int64)
    if kv.page_table is None:
        return b * int(kv.max_seq_len) + t
    P = int(kv.page_size)
    return kv.page_table[b, t // P].astype(np.int64) * P + t % P


def prefix_keys(kv, b: int, hk: int, dtype: str, tokens=None):
    """K, V [n, d] float64 of kv head hk of sequence b (all tokens, or a subset)."""
    slots = token_slots(kv, b)
    if tokens is not None:
        slots = slots[np.asarray(tokens, dtype=np.int64)]
    return to_f64(kv.k[slots, hk], dtype), to_f64(kv.v[slots, hk], dtype)


def prefix_partial(kv, q, dtype: str, scale: float = 1.0, head_mask=None):
    """(A_out, L_out) of every block row and q head over the block-external keys.

    q: [batch, B, Hq, d] storage array. q head h reads kv head h // (Hq/Hkv).
    head_mask [batch, Hq] (optional): heads with mask 0 are left as NaN.
    """
    batch, B, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    qf = to_f64(q, dtype)
    A = np.full((batch, B, Hq, d), np.nan)
    L = np.full((batch, B, Hq), np.nan)
    for b in range(batch):
        for hk in range(Hkv):
            heads = [hk * G + g for g in range(G)
                     if head_mask is None or head_mask[b, hk * G + g]]
            if not heads:
                continue
            K, V = prefix_keys(kv, b, hk, dtype)
            rows = qf[b][:, heads, :].reshape(-1, d)  # row r = i * len(heads) + g
            a, l = partial(rows, K, V, scale)
            A[b][:, heads, :] = a.reshape(B, len(heads), d)
            L[b][:, heads] = l.reshape(B, len(heads))
    return A, L


def prefix_partial_samples(kv, q, dtype: str, samples, scale: float = 1.0):
    """(A_out, L_out) for selected (b, i, h) rows only: [n, d], [n]."""
    Hq = q.shape[2]
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    out_A = np.zeros((len(samples), q.shape[3]))
    out_L = np.zeros(len(samples))
    by_head = {}
    for n, (b, i, h) in enumerate(samples):
        by_head.setdefault((b, h // G), []).append(n)
    for (b, hk), idx in by_head.items():
        K, V = prefix_keys(kv, b, hk, dtype)
        rows = np.stack([to_f64(q[samples[n][0], samples[n][1], samples[n][2]], dtype)
                         for n in idx])
        a, l = partial(rows, K, V, scale)
        out_A[idx] = a
        out_L[idx] = l
    return out_A, out_L


def block_partial(q, k_in, v_in, dtype: str, scale: float = 1.0):
    """(A_in, L_in): every block row against all B block tokens (bidirectional).

    q [batch, B, Hq, d], k_in / v_in [batch, B, Hkv, d] storage arrays.
    """
    batch, B, Hq, d = q.shape
    Hkv = k_in.shape[2]
    G = Hq // Hkv
    qf, kf, vf = to_f64(q, dtype), to_f64(k_in, dtype), to_f64(v_in, dtype)
    A = np.zeros((batch, B, Hq, d))
    L = np.zeros((batch, B, Hq))
    for b in range(batch):
        for h in range(Hq):
            a, l = partial(qf[b, :, h], kf[b, :, h // G], vf[b, :, h // G], scale)
            A[b, :, h] = a
            L[b, :, h] = l
    return A, L


def dense_attention(kv, q, k_in, v_in, dtype: str, scale: float = 1.0, samples=None):
    """Unsplit softmax attention over [prefix ; block], computed in one partial.

    This is the dense block-diffusion attention that FlashBlock decomposes; it
    never uses the merge, so it pins the merge from outside.
    Returns A [batch, B, Hq, d], L [batch, B, Hq] (or [n, d], [n] for samples).
    """
    batch, B, Hq, d = q.shape
    Hkv = kv.k.shape[1]
    G = Hq // Hkv
    if samples is None:
        samples = [(b, i, h) for b in range(batch) for i in range(B) for h in range(Hq)]
        full = True
    else:
        full = False
    out_A = np.zeros((len(samples), d))
    out_L = np.zeros(len(samples))
    by_head = {}
    for n, (b, i, h) in enumerate(samples):
        by_head.setdefault((b, h), []).append(n)
    for (b, h), idx in by_head.items():
        K, V = prefix_keys(kv, b, h // G, dtype)
        K = np.concatenate([K, to_f64(k_in[b, :, h // G], dtype)])
        V = np.concatenate([V, to_f64(v_in[b, :, h // G], dtype)])
        rows = to_f64(q[b, [samples[n][1] for n in idx], h], dtype)
        a, l = partial(rows, K, V, scale)
        out_A[idx] = a
        out_L[idx] = l
    if full:
        return out_A.reshape(batch, B, Hq, d), out_L.reshape(batch, B, Hq)
    return out_A, out_L
