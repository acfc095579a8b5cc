"""Workload specs and the seeded generator.

Five workloads stand in for the pages' models (the FlashBlock pages evaluate
Trado-8B/4B dLLMs and the LongLive-1.3B video model, the LoSA page Trado/SDAR
with block sizes 16/32); none of their weights or datasets are used. Shapes,
value distributions and update statistics are synthetic and seeded:

* ``tiny``  fp32, H=4, d=64, prefix 1024, block 16, 8 steps, tau=3; each step a
  random subset of Uniform{0..4} rows gets N(0, 0.5) added to its q/k/v.
* ``dllm``  bf16, batch 1, 32 heads MHA, d=128, prefix 32768, block 32, 32
  steps, tau=4; per step Poisson(2) rows are redrawn from N(0,1), every other
  row gets N(0, 0.02) jitter; K channels scaled by LogNormal(0, 0.5).
* ``gqa``   bf16, batch 8, 32 q heads / 8 kv heads, d=128, prefix lengths
  Uniform[16384, 65536] per sequence in a paged pool (page 16, pages permuted),
  block 64, 64 steps, Poisson(3) updates, tau=6, otherwise as ``dllm``.
* ``video`` bf16, 24 heads, d=128, block 1560 (one 30x52 latent frame), prefix
  32760 (21 frames), 50 steps, per-head input drift N(0, sigma_h) with sigma_h
  ~ Uniform[0.01, 0.3], gamma=0.95.
* ``losa``  bf16, 32 heads, d=128, prefix 131072 in pages of 16, block 32,
  |A|=4 active rows, top-256 pages, 32 steps, updates as ``dllm``.

N(mu, s) always names the standard deviation s. q is stored pre-scaled by
1/sqrt(d); kernels and oracle are then called with scale = 1.
"""

from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Iterator, Optional

import numpy as np

# Generation chunk (elements) for the prefix; fixed so values never depend on
# how the chunks are scheduled.
_CHUNK_ELEMS = 1 << 20
# bf16 bit pattern written into pool slots that no sequence owns (quiet NaN):
# any kernel that lets such a slot reach an output is caught by the tests.
BF16_NAN_BITS = 0x7FC0


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    return _round_bits_inplace(u).astype(np.uint16)


def _round_bits_inplace(u: np.ndarray) -> np.ndarray:
    """In place: float32 bit patterns -> bf16 bit patterns (still in uint32)."""
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    u += lsb
    u += np.uint32(0x7FFF)
    u >>= np.uint32(16)
    return u


@dataclass(frozen=True)
class Spec:
    name: str
    index: int
    dtype: str  # "f32" or "bf16"
    batch: int
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    block: int  # B, tokens in the block being denoised
    steps: int  # denoise steps for the block
    prefix_min: int  # prefix length bounds per sequence (inclusive)
    prefix_max: int
    page_size: int  # tokens per logical page of the prefix
    paged: bool  # True: permuted page pool + page table; False: contiguous slab
    update: str  # "subset" | "poisson" | "drift"
    rate: float  # subset: max rows per step; poisson: mean rows per step
    perturb_std: float  # subset: std of the additive perturbation
    jitter_std: float  # poisson: std of the jitter on non-redrawn rows
    k_scale_sigma: float  # LogNormal sigma of per-channel K scale (0: none)
    drift_lo: float = 0.0  # drift: per-head std ~ Uniform[drift_lo, drift_hi]
    drift_hi: float = 0.0
    tau: Optional[int] = None
    gamma: Optional[float] = None
    n_active: Optional[int] = None
    topk_pages: Optional[int] = None

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def group(self) -> int:
        return self.n_heads_q // self.n_heads_kv

    def with_(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


SPECS = {
    "tiny": Spec("tiny", 0, "f32", 1, 4, 4, 64, 16, 8, 1024, 1024, 16, False,
                 "subset", 4, 0.5, 0.0, 0.0, tau=3),
    "dllm": Spec("dllm", 1, "bf16", 1, 32, 32, 128, 32, 32, 32768, 32768, 16, False,
                 "poisson", 2.0, 0.0, 0.02, 0.5, tau=4),
    "gqa": Spec("gqa", 2, "bf16", 8, 32, 8, 128, 64, 64, 16384, 65536, 16, True,
                "poisson", 3.0, 0.0, 0.02, 0.5, tau=6),
    "video": Spec("video", 3, "bf16", 1, 24, 24, 128, 1560, 50, 32760, 32760, 16, False,
                  "drift", 0.0, 0.0, 0.0, 0.0, drift_lo=0.01, drift_hi=0.3, gamma=0.95),
    "losa": Spec("losa", 4, "bf16", 1, 32, 32, 128, 32, 32, 131072, 131072, 16, False,
                 "poisson", 2.0, 0.0, 0.02, 0.5, n_active=4, topk_pages=256),
}


@dataclass
class Prefix:
    """The frozen block-external KV cache (J_out) of every sequence.

    k, v: [n_slots, n_heads_kv, head_dim] storage arrays (float32, or uint16
    bf16 bits). Sequence b's token t lives in slot
      page_table[b, t // page_size] * page_size + t % page_size   (paged)
      b * max_seq_len + t                                          (contiguous)
    """

    k: np.ndarray
    v: np.ndarray
    seq_len: np.ndarray  # int32 [batch]
    page_table: Optional[np.ndarray]  # int32 [batch, max_pages] or None
    page_size: int
    max_seq_len: int

    @property
    def max_pages(self) -> int:
        return -(-self.max_seq_len // self.page_size)

    def slots(self, b: int) -> np.ndarray:
        """Slot index of every token of sequence b, in token order."""
        n = int(self.seq_len[b])
        t = np.arange(n, dtype=np.int64)
        if self.page_table is None:
            return b * self.max_seq_len + t
        pages = self.page_table[b, t // self.page_size].astype(np.int64)
        return pages * self.page_size + t % self.page_size


def grow_capacity(prefix: Prefix, extra_tokens: int, seed: int = 0) -> Prefix:
    """A copy of `prefix` with room for `extra_tokens` more tokens per sequence
    (layout only: no value is computed). Paged pools get the extra logical
    pages of every sequence mapped to new physical pages appended to the pool
    in a seeded permutation; contiguous pools get a longer per-sequence stride.
    New slots hold NaN (f32) / the bf16 NaN pattern, so a write that misses its
    slot is caught by any comparison."""
    P = int(prefix.page_size)
    batch = len(prefix.seq_len)
    new_max = int(prefix.max_seq_len) + int(extra_tokens)
    hd = prefix.k.shape[1:]
    fill = np.float32(np.nan) if prefix.k.dtype == np.float32 else np.uint16(BF16_NAN_BITS)
    if prefix.page_table is None:
        k = np.full((batch * new_max,) + hd, fill, dtype=prefix.k.dtype)
        v = np.full((batch * new_max,) + hd, fill, dtype=prefix.v.dtype)
        for b in range(batch):
            n = int(prefix.seq_len[b])
            src = b * int(prefix.max_seq_len)
            k[b * new_max: b * new_max + n] = prefix.k[src: src + n]
            v[b * new_max: b * new_max + n] = prefix.v[src: src + n]
        return Prefix(k, v, prefix.seq_len.copy(), None, P, new_max)
    old_pages = prefix.k.shape[0] // P
    have = [-(-int(n) // P) for n in prefix.seq_len]
    need = [-(-(int(n) + int(extra_tokens)) // P) for n in prefix.seq_len]
    total_new = int(sum(nd - hv for nd, hv in zip(need, have)))
    perm = old_pages + np.random.default_rng([seed, 11]).permutation(total_new).astype(np.int32)
    max_pages = -(-new_max // P)
    table = np.full((batch, max_pages), -1, dtype=np.int32)
    table[:, : prefix.page_table.shape[1]] = prefix.page_table
    off = 0
    for b in range(batch):
        cnt = need[b] - have[b]
        table[b, have[b]: need[b]] = perm[off: off + cnt]
        off += cnt
    pad = np.full((total_new * P,) + hd, fill, dtype=prefix.k.dtype)
    return Prefix(np.concatenate([prefix.k, pad]), np.concatenate([prefix.v, pad]),
                  prefix.seq_len.copy(), table, P, new_max)


@dataclass
class StepInputs:
    step: int
    q: np.ndarray  # [batch, B, Hq, d]
    k_in: np.ndarray  # [batch, B, Hkv, d]
    v_in: np.ndarray  # [batch, B, Hkv, d]
    m_updated: np.ndarray  # int32 [batch]: rows redrawn/perturbed since the last step


class Workload:
    """A seeded workload: the prefix plus an iterator over denoise steps."""

    def __init__(self, spec: Spec):
        self.spec = spec
        self.prefix = self._make_prefix()

    # -- storage helpers -------------------------------------------------
    def _store(self, x32: np.ndarray) -> np.ndarray:
        if self.spec.dtype == "f32":
            return np.ascontiguousarray(x32, dtype=np.float32)
        return bf16_bits_from_f32(x32)

    def _k_scale(self) -> np.ndarray:
        sp = self.spec
        rng = np.random.default_rng([sp.seed, 2])
        if sp.k_scale_sigma <= 0:
            return np.ones((sp.n_heads_kv, sp.head_dim), dtype=np.float32)
        return rng.lognormal(0.0, sp.k_scale_sigma,
                             size=(sp.n_heads_kv, sp.head_dim)).astype(np.float32)

    # -- prefix ----------------------------------------------------------
    def _make_prefix(self) -> Prefix:
        sp = self.spec
        rng = np.random.default_rng([sp.seed, 0])
        if sp.prefix_min == sp.prefix_max:
            seq_len = np.full(sp.batch, sp.prefix_min, dtype=np.int32)
        else:
            seq_len = rng.integers(sp.prefix_min, sp.prefix_max, endpoint=True,
                                   size=sp.batch).astype(np.int32)
        max_len = int(sp.prefix_max)
        P = sp.page_size
        kscale = self._k_scale()
        hd = (sp.n_heads_kv, sp.head_dim)
        if sp.paged:
            n_pages = [-(-int(n) // P) for n in seq_len]
            total = int(sum(n_pages))
            perm = rng.permutation(total).astype(np.int32)
            max_pages = -(-max_len // P)
            table = np.full((sp.batch, max_pages), -1, dtype=np.int32)
            off = 0
            for b, npg in enumerate(n_pages):
                table[b, :npg] = perm[off:off + npg]
                off += npg
            n_slots = total * P
        else:
            table = None
            n_slots = sp.batch * max_len
        sdt = np.float32 if sp.dtype == "f32" else np.uint16
        fill = np.float32(np.nan) if sp.dtype == "f32" else np.uint16(BF16_NAN_BITS)
        if sp.paged or int(seq_len.min()) < max_len:
            k = np.full((n_slots,) + hd, fill, dtype=sdt)
            v = np.full((n_slots,) + hd, fill, dtype=sdt)
        else:  # every slot is owned by a token and written below
            k = np.empty((n_slots,) + hd, dtype=sdt)
            v = np.empty((n_slots,) + hd, dtype=sdt)
        pre = Prefix(k, v, seq_len, table, P, max_len)
        ct = max(P, _CHUNK_ELEMS // (sp.n_heads_kv * sp.head_dim) // P * P)
        jobs = [(b, t0) for b in range(sp.batch)
                for t0 in range(0, int(seq_len[b]), ct)]
        slots_of = [pre.slots(b) for b in range(sp.batch)]

        def fill(job):
            # every chunk has its own substream, so chunks can be drawn in any
            # order (and in parallel) with identical values
            b, t0 = job
            crng = np.random.default_rng([sp.seed, 3, b, t0 // ct])
            t1 = min(int(seq_len[b]), t0 + ct)
            x = np.empty((t1 - t0,) + hd, dtype=np.float32)
            for dst, sc in ((k, kscale), (v, None)):
                crng.standard_normal(out=x, dtype=np.float32)
                if sc is not None:
                    x *= sc
                y = _round_bits_inplace(x.copy().view(np.uint32)) if sp.dtype == "bf16" else x
                if pre.page_table is None:
                    base = b * max_len
                    np.copyto(dst[base + t0: base + t1], y, casting="unsafe")
                else:  # whole pages first (one index per page), then the ragged tail
                    yy = y.astype(sdt, copy=False)
                    nfull = (t1 - t0) // P
                    pages = pre.page_table[b, t0 // P: t0 // P + nfull]
                    dst.reshape((-1, P) + hd)[pages] = yy[: nfull * P].reshape((nfull, P) + hd)
                    if nfull * P < t1 - t0:
                        dst[slots_of[b][t0 + nfull * P: t1]] = yy[nfull * P:]

        with ThreadPoolExecutor(max_workers=int(os.environ.get("FB_GEN_THREADS", min(8, os.cpu_count() or 1)))) as ex:
            list(ex.map(fill, jobs))
        return pre

    # -- denoise steps -----------------------------------------------------
    def steps(self, n_steps: Optional[int] = None) -> Iterator[StepInputs]:
        """Yield the block's inputs for steps 0..n_steps-1 (default: spec.steps)."""
        sp = self.spec
        n_steps = sp.steps if n_steps is None else n_steps
        rng = np.random.default_rng([sp.seed, 1])
        B, Hq, Hkv, d = sp.block, sp.n_heads_q, sp.n_heads_kv, sp.head_dim
        kscale = self._k_scale()
        qscale = np.float32(1.0 / math.sqrt(d))
        sigma = None
        if sp.update == "drift":
            sigma = rng.uniform(sp.drift_lo, sp.drift_hi, size=Hq).astype(np.float32)
        shp_q = (sp.batch, B, Hq, d)
        shp_kv = (sp.batch, B, Hkv, d)
        q = rng.standard_normal(shp_q, dtype=np.float32)
        kr = rng.standard_normal(shp_kv, dtype=np.float32)
        vr = rng.standard_normal(shp_kv, dtype=np.float32)
        m = np.full(sp.batch, B, dtype=np.int32)
        for s in range(n_steps):
            if s > 0:
                m = self._update(rng, q, kr, vr, sigma)
            yield StepInputs(s, self._store(q * qscale), self._store(kr * kscale),
                             self._store(vr), m.copy())

    def _update(self, rng, q, kr, vr, sigma) -> np.ndarray:
        """Advance the raw (unscaled) block state by one denoise step in place."""
        sp = self.spec
        B = sp.block
        m = np.zeros(sp.batch, dtype=np.int32)
        if sp.update == "drift":
            # every row drifts; the per-head std applies to q, k and v of head h
            # (MHA here, so q head h and kv head h coincide).
            q += rng.standard_normal(q.shape, dtype=np.float32) * sigma[None, None, :, None]
            sk = sigma.reshape(sp.n_heads_kv, sp.group).mean(axis=1)
            kr += rng.standard_normal(kr.shape, dtype=np.float32) * sk[None, None, :, None]
            vr += rng.standard_normal(vr.shape, dtype=np.float32) * sk[None, None, :, None]
            m[:] = B
            return m
        for b in range(sp.batch):
            if sp.update == "subset":
                cnt = int(rng.integers(0, int(sp.rate), endpoint=True))
                rows = rng.choice(B, size=cnt, replace=False)
                for x in (q, kr, vr):
                    x[b, rows] += rng.standard_normal(x[b, rows].shape,
                                                      dtype=np.float32) * np.float32(sp.perturb_std)
            elif sp.update == "poisson":
                cnt = min(int(rng.poisson(sp.rate)), B)
                rows = rng.choice(B, size=cnt, replace=False)
                keep = np.ones(B, dtype=bool)
                keep[rows] = False
                for x in (q, kr, vr):
                    x[b, rows] = rng.standard_normal(x[b, rows].shape, dtype=np.float32)
                    x[b, keep] += rng.standard_normal(x[b, keep].shape,
                                                      dtype=np.float32) * np.float32(sp.jitter_std)
            else:
                raise ValueError(sp.update)
            m[b] = cnt
        return m


def make_workload(name: str, **overrides) -> Workload:
    """Build a workload by name; keyword overrides shrink it for tests."""
    return Workload(SPECS[name].with_(**overrides))
