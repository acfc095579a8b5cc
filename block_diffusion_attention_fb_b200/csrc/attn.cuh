// Attention partials (A, L = log Z) of block query rows over a key set, the
// split-KV combine, and the FlashBlock log-space merge.
//
// One kernel family serves three key sets (FlashBlock technical summary, §2
// "Core mechanism"; LoSA, §2 step 3):
//   * the block-external prefix J_out (contiguous or paged cache),
//   * the block's own tokens J_in (bidirectional, contiguous),
//   * the union of LoSA-selected pages of a kv head (page list).
// A CTA owns (sequence b, kv head hk, key split, row tile). Its rows are the
// block rows taking part times the G q heads sharing hk (GQA stacking), so a
// K/V tile read from HBM once serves every q head of the group.
//
// bf16 path: one producer warp streams K/V tiles of kTK keys with TMA
// (128-byte swizzle, 3-stage mbarrier pipeline); four consumer warps run
// QK^T and PV on bf16 tensor cores (mma.sync m16n8k16, fp32 accumulate) with
// ldmatrix fragment loads and an online softmax in registers (exp2 domain).
// Consumer warps split the tile's keys (RG row groups x KS key slices) and
// merge their partial softmax states through shared memory at the end.
// f32 path: CUDA-core FMA (the fp32 workloads are launch-bound).
#pragma once

#include "common.cuh"

namespace fb {

constexpr int kTK = 64;      // keys per pipeline stage / tile
constexpr int kStages = 3;   // TMA pipeline depth
constexpr int kNWC = 4;      // consumer warps per CTA (bf16)
constexpr int kAttnThreads = (kNWC + 1) * 32;
constexpr int kMaxChunks = kTK / 16;  // TMA boxes per tile and half (page >= 16)
constexpr int kSlotAhead = 3;  // tiles whose chunk slots a producer fetches ahead
constexpr int kSlotRing = kSlotAhead + 1;

struct AttnArgs {
  const void* q;  // [batch, B, Hq, D], or [q_total, Hq, D] packed (q_cu)
  const void* k;  // [n_slots, Hkv, D] (f32 path; the bf16 path reads through TMA)
  const void* v;
  int batch, B, Hq, Hkv, G;  // B: rows per sequence (packed rows: the most any sequence has)
  // Packed (variable-length) rows: sequence b's query rows are rows
  // q_cu[b] .. q_cu[b+1]-1 of q and of the outputs; NULL: rows b * B + i.
  const int32_t* q_cu;
  int q_total;  // rows of the packed buffers
  // Packed contiguous key set (a varlen block's own keys): sequence b's tokens
  // are rows kv_cu[b] .. kv_cu[b+1]-1 of k / v; NULL: the cache layout below.
  const int32_t* kv_cu;
  const int32_t* row_list;  // [batch, n_list] block rows taking part, or NULL (all B)
  int n_list;
  int R;  // rows per (b, hk): (row_list ? n_list : B) * G; row r = i_idx * G + g
  int row_tile, n_row_tiles;
  // key set
  const int32_t* page_table;  // [batch, max_pages] or NULL (contiguous)
  int max_pages, page_size;
  const int32_t* seq_len;  // [batch] or NULL (all max_seq_len)
  int max_seq_len;
  const int32_t* page_list;   // [batch, Hkv, page_list_stride] or NULL (dense key set)
  const int32_t* page_count;  // [batch, Hkv]
  int page_list_stride;
  int chunk;  // tokens per TMA box / metadata chunk: kTK (contiguous dense) or min(page, kTK)
  long long n_slots;
  // which heads compute
  const uint8_t* head_mask;  // [batch, Hq] or NULL
  unsigned long long seq_bits[4];
  int use_seq_bits;
  // split plan
  int tiles_per_split, n_splits;
  float scale_log2;  // softmax scale * log2(e)
  // outputs: split partials (n_splits > 1) or final rows (n_splits == 1)
  float* o_part;    // [n_splits, batch, Hkv, R, D] normalised partial outputs
  float* lse_part;  // [n_splits, batch, Hkv, R] log2 normalisers (-inf: empty)
  float* a_out;     // [batch, B, Hq, D]
  float* l_out;     // [batch, B, Hq] natural log
  float* a_prev;    // optional: old a_out rows are copied here before overwrite
  const float* mrg_a;  // optional second partial merged into every final row (FlashBlock merge)
  const float* mrg_l;
};

__device__ __forceinline__ int seq_tokens(const AttnArgs& a, int b) {
  if (a.kv_cu) {
    long long t0;
    return packed_range(a.kv_cu, b, (int)a.n_slots, a.max_seq_len, t0);
  }
  return a.seq_len ? a.seq_len[b] : a.max_seq_len;
}

// First output row of sequence b and its stacked row count (block rows x G).
__device__ __forceinline__ long long q_row0(const AttnArgs& a, int b) {
  if (!a.q_cu) return (long long)b * a.B;
  long long r0;
  packed_range(a.q_cu, b, a.q_total, a.B, r0);
  return r0;
}
__device__ __forceinline__ int rows_of(const AttnArgs& a, int b) {
  if (!a.q_cu) return a.R;
  long long r0;
  return packed_range(a.q_cu, b, a.q_total, a.B, r0) * a.G;
}

__device__ __forceinline__ bool cta_selected(const AttnArgs& a, int b, int hk) {
  if (a.use_seq_bits && !((a.seq_bits[b >> 6] >> (b & 63)) & 1ull)) return false;
  if (a.head_mask) {
    for (int g = 0; g < a.G; ++g)
      if (a.head_mask[b * a.Hq + hk * a.G + g]) return true;
    return false;
  }
  return true;
}

__device__ __forceinline__ bool row_selected(const AttnArgs& a, int b, int h) {
  if (a.use_seq_bits && !((a.seq_bits[b >> 6] >> (b & 63)) & 1ull)) return false;
  return a.head_mask == nullptr || a.head_mask[b * a.Hq + h] != 0;
}

// Number of kTK-key tiles of (b, hk)'s key set.
__device__ __forceinline__ int n_tiles_of(const AttnArgs& a, int b, int hk) {
  if (a.page_list) {
    const int per_tile = kTK / a.page_size;
    const int cnt = a.page_count[b * a.Hkv + hk];
    return (cnt + per_tile - 1) / per_tile;
  }
  return (seq_tokens(a, b) + kTK - 1) / kTK;
}

// Slot of the first token of chunk c of tile tl, and how many of the chunk's
// tokens are valid (0 => the chunk is loaded out of bounds, i.e. zero-filled).
// Per-(sequence, kv head) values every chunk lookup needs, read once per CTA
// (a producer would otherwise pay a global load on every tile).
struct GroupInfo {
  int n_tok;       // tokens of the sequence
  int list_cnt;    // entries of the page list (page-list key sets)
  long long base;  // contiguous key sets: pool row of the sequence's first token
};

__device__ __forceinline__ GroupInfo group_info(const AttnArgs& a, int b, int hk) {
  GroupInfo g;
  g.base = (long long)b * a.max_seq_len;
  if (a.kv_cu)
    g.n_tok = packed_range(a.kv_cu, b, (int)a.n_slots, a.max_seq_len, g.base);
  else
    g.n_tok = a.seq_len ? a.seq_len[b] : a.max_seq_len;
  g.list_cnt = a.page_list ? a.page_count[b * a.Hkv + hk] : 0;
  return g;
}

// n_tiles_of from the values group_info already read
__device__ __forceinline__ int n_tiles_of(const AttnArgs& a, const GroupInfo& gi) {
  if (a.page_list) {
    const int per_tile = kTK / a.page_size;
    return (gi.list_cnt + per_tile - 1) / per_tile;
  }
  return (gi.n_tok + kTK - 1) / kTK;
}

__device__ __forceinline__ void chunk_slot(const AttnArgs& a, const GroupInfo& gi, int b, int hk,
                                           int tl, int c, long long& slot, int& valid) {
  const int n_tok = gi.n_tok;
  int t0;
  if (a.page_list) {
    const int per_tile = kTK / a.page_size;
    const int e = tl * per_tile + c;
    if (e >= gi.list_cnt) {
      slot = a.n_slots;
      valid = 0;
      return;
    }
    const int lp = a.page_list[((long long)b * a.Hkv + hk) * a.page_list_stride + e];
    t0 = lp * a.page_size;
  } else {
    t0 = tl * kTK + c * a.chunk;
  }
  valid = min(max(n_tok - t0, 0), a.chunk);
  if (valid == 0) {
    slot = a.n_slots;
    return;
  }
  if (a.page_table) {
    const int lp = t0 / a.page_size;
    const int off = t0 - lp * a.page_size;
    const int pg = a.page_table[(long long)b * a.max_pages + lp];
    if (pg < 0 || ((long long)pg + 1) * a.page_size > a.n_slots) {
      // an entry outside the pool: the chunk reads as holding no tokens (no
      // access is made through it) and the error word records it
      atomicOr(&g_fb_error_word, kErrBadReadPage);
      slot = a.n_slots;
      valid = 0;
      return;
    }
    slot = (long long)pg * a.page_size + off;
  } else {
    slot = gi.base + t0;
  }
}

__device__ __forceinline__ void chunk_slot(const AttnArgs& a, int b, int hk, int tl, int c,
                                           long long& slot, int& valid) {
  chunk_slot(a, group_info(a, b, hk), b, hk, tl, c, slot, valid);
}

// Key tiles per split of (b, hk). Dense key sets use the plan's; page lists,
// whose lengths the host plan only bounds, spread their actual tiles evenly
// over the planned splits (no more than the plan's, so every buffer sized by
// the plan still holds). even: a whole number of 128-key tiles (tcgen05).
__device__ __forceinline__ int split_tiles(const AttnArgs& a, int n_tiles, bool even) {
  if (!a.page_list) return a.tiles_per_split;
  int t = (n_tiles + a.n_splits - 1) / a.n_splits;
  if (even) t = (t + 1) & ~1;
  return min(max(t, even ? 2 : 1), a.tiles_per_split);
}

// Maps row r of (b, hk) to the block row i and q head h.
__device__ __forceinline__ void row_of(const AttnArgs& a, int b, int hk, int r, int& i, int& h) {
  const int i_idx = r / a.G;
  h = hk * a.G + (r - i_idx * a.G);
  i = a.row_list ? a.row_list[b * a.n_list + i_idx] : i_idx;
}

// Writes one final row: vals (normalised, NV per lane at col0 + j*col_stride)
// and lse2 (log2 units). With mrg_a set the row is first merged with the
// second partial by the FlashBlock rule: m = max(L1, L2), w_x = e^{L_x - m},
// A = (w1 A1 + w2 A2) / (w1 + w2), L = m + log(w1 + w2); a side with L = -inf
// is not read.
template <int NV>
__device__ __forceinline__ void write_final(const AttnArgs& a, int b, int hk, int r,
                                            const float (&val)[NV], int col0, int col_stride,
                                            float lse2, bool lane0) {
  int i, h;
  row_of(a, b, hk, r, i, h);
  if (!row_selected(a, b, h)) return;
  const long long row = (q_row0(a, b) + i) * a.Hq + h;
  constexpr int D = NV * 32;
  float* dst = a.a_out + row * D;
  const float Ln = lse2 * kLn2;
  float wn = 1.f, wo = 0.f, L = Ln;
  if (a.mrg_a) {
    const float Lo = a.mrg_l[row];
    const float m = fmaxf(Lo, Ln);
    if (m == -INFINITY) {
      wn = 0.f;
      L = -INFINITY;
    } else {
      const float eo = expf(Lo - m), en = expf(Ln - m);
      const float inv = 1.f / (eo + en);
      wn = en * inv;
      wo = eo * inv;
      L = m + logf(eo + en);
    }
  }
  if (a.a_prev) {
    float* prv = a.a_prev + row * D;
#pragma unroll
    for (int j = 0; j < NV; ++j) prv[col0 + j * col_stride] = dst[col0 + j * col_stride];
  }
  const float* old = a.mrg_a ? a.mrg_a + row * D : nullptr;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int col = col0 + j * col_stride;
    float v = wn > 0.f ? wn * val[j] : 0.f;
    if (old && wo > 0.f) v += wo * old[col];
    dst[col] = v;
  }
  if (lane0) a.l_out[row] = L;
}

// Writes one finished row: a split partial (n_splits > 1) or the final row.
template <int NV>
__device__ __forceinline__ void store_row(const AttnArgs& a, int b, int hk, int split, int r,
                                          const float (&val)[NV], int col0, int col_stride,
                                          float lse2, bool lane0) {
  if (a.n_splits > 1) {
    const long long pidx = (((long long)split * a.batch + b) * a.Hkv + hk) * a.R + r;
    float* dst = a.o_part + pidx * (NV * 32);
#pragma unroll
    for (int j = 0; j < NV; ++j) dst[col0 + j * col_stride] = val[j];
    if (lane0) a.lse_part[pidx] = lse2;
    return;
  }
  write_final<NV>(a, b, hk, r, val, col0, col_stride, lse2, lane0);
}

// write_final for RB rows of one warp at once: every global read the rows need
// (merge partner, old rows) is issued before any arithmetic or store, so the
// rows' memory latencies overlap instead of adding up.
template <int NV, int RB>
__device__ __forceinline__ void write_final_rows(const AttnArgs& a, int b, int hk,
                                                 const int (&r)[RB], const float (&val)[RB][NV],
                                                 const float (&lse2)[RB], int lane) {
  constexpr int D = NV * 32;
  long long row[RB];
  bool ok[RB];
  float Lo[RB], old[RB][NV], prv[RB][NV];
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    ok[k] = r[k] >= 0;
    row[k] = 0;
    if (ok[k]) {
      int i, h;
      row_of(a, b, hk, r[k], i, h);
      ok[k] = row_selected(a, b, h);
      row[k] = (q_row0(a, b) + i) * a.Hq + h;
    }
  }
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    Lo[k] = -INFINITY;
#pragma unroll
    for (int j = 0; j < NV; ++j) old[k][j] = prv[k][j] = 0.f;
    if (!ok[k]) continue;
    if (a.mrg_a) {
      Lo[k] = a.mrg_l[row[k]];
#pragma unroll
      for (int j = 0; j < NV; ++j) old[k][j] = a.mrg_a[row[k] * D + lane * NV + j];
    }
    if (a.a_prev) {
#pragma unroll
      for (int j = 0; j < NV; ++j) prv[k][j] = a.a_out[row[k] * D + lane * NV + j];
    }
  }
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    if (!ok[k]) continue;
    const float Ln = lse2[k] * kLn2;
    float wn = 1.f, wo = 0.f, L = Ln;
    if (a.mrg_a) {
      const float m = fmaxf(Lo[k], Ln);
      if (m == -INFINITY) {
        wn = 0.f;
        L = -INFINITY;
      } else {
        const float eo = expf(Lo[k] - m), en = expf(Ln - m);
        const float inv = 1.f / (eo + en);
        wn = en * inv;
        wo = eo * inv;
        L = m + logf(eo + en);
      }
    }
    if (a.a_prev) {
#pragma unroll
      for (int j = 0; j < NV; ++j) a.a_prev[row[k] * D + lane * NV + j] = prv[k][j];
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      float v = wn > 0.f ? wn * val[k][j] : 0.f;
      if (wo > 0.f) v += wo * old[k][j];
      a.a_out[row[k] * D + lane * NV + j] = v;
    }
    if (lane == 0) a.l_out[row[k]] = L;
  }
}

// Merges the n_splits partials of row r of (b, hk) (log-space rule) and writes
// the final row. One warp, NV contiguous columns per lane. The normalisers of
// 32 splits are read at once (one per lane) and their weights broadcast by
// shuffle, so the partial loads of a chunk are independent of each other.
// Every split writes its partial and normaliser, an empty one zeros and -inf;
// a split of weight exactly 0 is left out of the sum rather than multiplied by
// 0, so no value it holds (a NaN left in reused scratch included) reaches the
// row, while a NaN weight still propagates.
template <int NV>
__device__ __forceinline__ void combine_row(const AttnArgs& a, int b, int hk, int r, int lane) {
  constexpr int D = NV * 32;
  const long long stride = (long long)a.batch * a.Hkv * a.R;  // between splits
  const long long p0 = ((long long)b * a.Hkv + hk) * a.R + r;
  constexpr int kFast = 16;
  if (a.n_splits <= kFast) {
    // Up to 16 splits: every partial and normaliser load is issued before any
    // of them is used, so a row costs one memory round trip.
    float v[kFast][NV];
    const float l = lane < a.n_splits ? __ldcg(a.lse_part + p0 + lane * stride) : -INFINITY;
#pragma unroll
    for (int s = 0; s < kFast; ++s) {
      if (s < a.n_splits) {
        const float* src = a.o_part + (p0 + (long long)s * stride) * D + lane * NV;
        if constexpr (NV == 4) {
          const float4 t = __ldcg(reinterpret_cast<const float4*>(src));
          v[s][0] = t.x;
          v[s][1] = t.y;
          v[s][2] = t.z;
          v[s][3] = t.w;
        } else {
#pragma unroll
          for (int jj = 0; jj < NV; ++jj) v[s][jj] = __ldcg(src + jj);
        }
      }
    }
    float M = l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float bse = (M == -INFINITY) ? 0.f : M;
    const float wl = l == -INFINITY ? 0.f : fast_exp2(l - bse);
    float acc[NV], wsum = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) acc[j] = 0.f;
#pragma unroll
    for (int s = 0; s < kFast; ++s) {
      if (s < a.n_splits) {
        const float w = __shfl_sync(0xffffffffu, wl, s);
        wsum += w;
        if (w != 0.f) {
#pragma unroll
          for (int j = 0; j < NV; ++j) acc[j] += w * v[s][j];
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) acc[j] *= inv;
    const float lse2 = wsum > 0.f ? bse + log2f(wsum) : -INFINITY;
    write_final<NV>(a, b, hk, r, acc, lane * NV, 1, lse2, lane == 0);
    return;
  }
  float M = -INFINITY;
  for (int s = lane; s < a.n_splits; s += 32) M = fmaxf(M, __ldcg(a.lse_part + p0 + s * stride));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float bse = (M == -INFINITY) ? 0.f : M;
  float acc[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) acc[j] = 0.f;
  float wsum = 0.f;
  for (int s0 = 0; s0 < a.n_splits; s0 += 32) {
    const int s = s0 + lane;
    const float l = s < a.n_splits ? __ldcg(a.lse_part + p0 + s * stride) : -INFINITY;
    const float wl = l == -INFINITY ? 0.f : fast_exp2(l - bse);
    const int n = min(32, a.n_splits - s0);
#pragma unroll 8
    for (int j = 0; j < n; ++j) {
      const float w = __shfl_sync(0xffffffffu, wl, j);
      wsum += w;
      if (w != 0.f) {
        const float* src = a.o_part + (p0 + (long long)(s0 + j) * stride) * D + lane * NV;
        if constexpr (NV == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
          acc[0] += w * v.x;
          acc[1] += w * v.y;
          acc[2] += w * v.z;
          acc[3] += w * v.w;
        } else {
#pragma unroll
          for (int jj = 0; jj < NV; ++jj) acc[jj] += w * __ldcg(src + jj);
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) acc[j] *= inv;
  const float lse2 = wsum > 0.f ? bse + log2f(wsum) : -INFINITY;
  write_final<NV>(a, b, hk, r, acc, lane * NV, 1, lse2, lane == 0);
}

// ---------------------------------------------------------------------------
// bf16 tensor-core kernel
// ---------------------------------------------------------------------------
template <int D>
struct Bf16Smem {
  static constexpr int kHalves = D / 64;  // 128-byte swizzle rows hold 64 bf16
  static constexpr int kHalfBytes = kTK * 128;
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // K or V of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kRedStride = D + 4;  // padded fp32 row for the cross-warp merge
  static constexpr int kRedBytes = kNWC * 16 * kRedStride * 4 + 2 * kNWC * 16 * 4;
  static constexpr int kBytes =
      (kStages * kStageBytes > kRedBytes ? kStages * kStageBytes : kRedBytes) + 1024;
  static_assert(kRedBytes <= kStages * kStageBytes, "merge area must fit in the stages");
};

template <int D, int RG>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_bf16_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  using S = Bf16Smem<D>;
  constexpr int KS = kNWC / RG;   // key slices
  constexpr int KW = kTK / KS;    // keys per warp per tile
  constexpr int SUB = KW < 32 ? KW : 32;
  constexpr int NT = SUB / 8;     // n8 tiles per sub-chunk
  constexpr int KD = D / 16;      // k16 steps over the head dim

  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ int meta[kStages][kMaxChunks];
  __shared__ int meta_full[kStages];
  __shared__ int abort_flag;
  // chunk slots / valid counts of upcoming tiles, filled by the producer warp
  __shared__ int ring_slot[kSlotRing][kMaxChunks];
  __shared__ int ring_valid[kSlotRing][kMaxChunks];
  extern __shared__ uint8_t dyn_smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x % a.n_row_tiles;
  const int split = blockIdx.x / a.n_row_tiles;
  const int hk = blockIdx.y, b = blockIdx.z;
  if (!cta_selected(a, b, hk)) return;
  const int Rb = rows_of(a, b);  // stacked rows of this sequence
  if (rt * a.row_tile >= Rb) return;

  const int n_tiles = n_tiles_of(a, b, hk);
  const int tps = split_tiles(a, n_tiles, false);
  const int tile0 = split * tps;
  const int n_it = max(0, min(tps, n_tiles - tile0));
  const int n_chunks = kTK / a.chunk;

  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* base_ptr = dyn_smem + (base - smem_u32(dyn_smem));

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kNWC);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kNWC) {
    // ----------------------------- producer -----------------------------
    // Lane 0 waits for free stages and issues the copies; all lanes fetch the
    // chunk slots of the tile kSlotAhead tiles ahead (one chunk per lane) into
    // a shared ring, so page-list / page-table reads overlap earlier copies.
    const GroupInfo gi = group_info(a, b, hk);
    auto fill = [&](int it) {  // tile `it` -> ring entry it % kSlotRing (all lanes)
      if (lane < n_chunks) {
        long long s_ = a.n_slots;
        int v_ = 0;
        chunk_slot(a, gi, b, hk, tile0 + it, lane, s_, v_);
        ring_slot[it % kSlotRing][lane] = (int)s_;
        ring_valid[it % kSlotRing][lane] = v_;
      }
    };
    for (int it = 0; it < kSlotAhead && it < n_it; ++it) fill(it);
    __syncwarp();
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    int issued = 0;
    for (int it = 0; it < n_it; ++it) {
      // entry (it + kSlotAhead) % kSlotRing last served tile it - 1
      if (it + kSlotAhead < n_it) fill(it + kSlotAhead);
      int ok = 1;
      if (lane == 0) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int re = it % kSlotRing;
        ok = mbar_wait(&empty_bar[st], ph ^ 1, &abort_flag);
        if (ok) {
          int all_full = 1;
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            if (c < n_chunks) {
              meta[st][c] = ring_valid[re][c];
              all_full &= (ring_valid[re][c] == a.chunk);
            }
          }
          meta_full[st] = all_full;
          mbar_arrive_expect_tx(&full_bar[st], S::kStageBytes);
          uint8_t* sk = base_ptr + st * S::kStageBytes;
          uint8_t* sv = sk + S::kTileBytes;
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            if (c < n_chunks) {
              const int z = ring_slot[re][c];
#pragma unroll
              for (int hf = 0; hf < S::kHalves; ++hf) {
                uint8_t* dk = sk + hf * S::kHalfBytes + c * a.chunk * 128;
                uint8_t* dv = sv + hf * S::kHalfBytes + c * a.chunk * 128;
                tma_load_3d(dk, &tmK, hf * 64, hk, z, &full_bar[st]);
                tma_load_3d(dv, &tmV, hf * 64, hk, z, &full_bar[st]);
              }
            }
          }
          ++issued;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();  // ring entries written this iteration are visible to lane 0 next time
    }
    if (lane == 0 && abort_flag) {
      // let copies already in flight land before the CTA's memory goes away
      const long long t0 = clock64();
      for (int it = max(0, issued - kStages); it < issued; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        while (!mbar_try_wait(&full_bar[st], ph) && clock64() - t0 < kWaitBudgetCycles) {
        }
      }
    }
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int rg = warp % RG, ks = warp / RG;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int row_base = rt * a.row_tile + rg * 16;

  // Q fragments (A operand of QK^T), rows g8 and g8 + 8 of this row group.
  uint32_t qa[KD][4];
  {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q);
    const __nv_bfloat16* rowp[2] = {nullptr, nullptr};
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = row_base + g8 + hr * 8;
      if (r < Rb) {
        int i, h;
        row_of(a, b, hk, r, i, h);
        rowp[hr] = qb + ((q_row0(a, b) + i) * a.Hq + h) * D;
      }
    }
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int hr = j & 1;
        const int col = kk * 16 + (j >> 1) * 8 + 2 * t4;
        qa[kk][j] = rowp[hr] ? *reinterpret_cast<const uint32_t*>(rowp[hr] + col) : 0u;
      }
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.f, 0.f};

  const int mi = lane >> 3, r8 = lane & 7;
  for (int it = 0; it < n_it; ++it) {
    const int st = it % kStages;
    const uint32_t ph = (it / kStages) & 1;
    if (!mbar_wait(&full_bar[st], ph, &abort_flag)) break;
    const uint32_t sK = base + st * S::kStageBytes;
    const uint32_t sV = sK + S::kTileBytes;
    const bool tile_full = meta_full[st] != 0;
    const int chunk = a.chunk;
    bool wrote_smem = false;

#pragma unroll
    for (int sub = 0; sub < KW / SUB; ++sub) {
      const int kb = ks * KW + sub * SUB;  // first key of this sub-chunk in the tile
      float s[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const int key = kb + np * 16 + (mi >> 1) * 8 + r8;
          const int ch = 2 * kk + (mi & 1);
          const uint32_t addr =
              sK + (ch >> 3) * S::kHalfBytes + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16(s[2 * np], qa[kk], b0, b1);
          mma_bf16(s[2 * np + 1], qa[kk], b2, b3);
        }
      }
      // scale into the exp2 domain and mask keys outside the key set
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] *= a.scale_log2;
      if (!tile_full) {
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = kb + n * 8 + 2 * t4 + (e & 1);
            const int c = key / chunk;
            if (key - c * chunk >= meta[st][c]) s[n][e] = -INFINITY;
          }
        // V rows of masked keys may hold any bits: zero them so p = 0 stays 0
        for (int idx = lane; idx < SUB * (D / 8); idx += 32) {
          const int kr = idx / (D / 8), ch = idx % (D / 8);
          const int key = kb + kr;
          const int c = key / chunk;
          if (key - c * chunk >= meta[st][c]) {
            uint8_t* p = base_ptr + (sV - base) + (ch >> 3) * S::kHalfBytes + key * 128 +
                         (((ch & 7) ^ (key & 7)) << 4);
            *reinterpret_cast<uint4*>(p) = make_uint4(0u, 0u, 0u, 0u);
            wrote_smem = true;
          }
        }
        __syncwarp();
      }
      // online softmax (rows g8 and g8 + 8)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
        mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
      }
      float alpha[2], bse[2];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
        const float mn = fmaxf(m_r[hr], mx[hr]);
        bse[hr] = (mn == -INFINITY) ? 0.f : mn;
        alpha[hr] = fast_exp2(m_r[hr] - bse[hr]);
        m_r[hr] = mn;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s[n][e] = fast_exp2(s[n][e] - bse[e >> 1]);
          rs[e >> 1] += s[n][e];
        }
      }
      l_r[0] = l_r[0] * alpha[0] + rs[0];
      l_r[1] = l_r[1] * alpha[1] + rs[1];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
      // O += P V
#pragma unroll
      for (int kst = 0; kst < SUB / 16; ++kst) {
        const uint32_t pa[4] = {pack_bf16(s[2 * kst][0], s[2 * kst][1]),
                                pack_bf16(s[2 * kst][2], s[2 * kst][3]),
                                pack_bf16(s[2 * kst + 1][0], s[2 * kst + 1][1]),
                                pack_bf16(s[2 * kst + 1][2], s[2 * kst + 1][3])};
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          const int key = kb + kst * 16 + (mi & 1) * 8 + r8;
          const int ch = 2 * dp + (mi >> 1);
          const uint32_t addr =
              sV + (ch >> 3) * S::kHalfBytes + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16(o[2 * dp], pa, b0, b1);
          mma_bf16(o[2 * dp + 1], pa, b2, b3);
        }
      }
    }
    if (wrote_smem) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);
  }

  // --------------------- cross-warp merge and output ----------------------
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
    l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
  }
  named_bar_sync(1, kNWC * 32);  // every consumer is done with the stage buffers
  float* redO = reinterpret_cast<float*>(base_ptr);
  float* redM = redO + kNWC * 16 * S::kRedStride;
  float* redL = redM + kNWC * 16;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * t4;
    *reinterpret_cast<float2*>(&redO[(warp * 16 + g8) * S::kRedStride + col]) =
        make_float2(o[n][0], o[n][1]);
    *reinterpret_cast<float2*>(&redO[(warp * 16 + g8 + 8) * S::kRedStride + col]) =
        make_float2(o[n][2], o[n][3]);
  }
  if (t4 == 0) {
    redM[warp * 16 + g8] = m_r[0];
    redM[warp * 16 + g8 + 8] = m_r[1];
    redL[warp * 16 + g8] = l_r[0];
    redL[warp * 16 + g8 + 8] = l_r[1];
  }
  named_bar_sync(1, kNWC * 32);
  constexpr int NV = D / 32;
  constexpr int RB = (RG * 16) / kNWC < 4 ? (RG * 16) / kNWC : 4;  // rows per batch of a warp
  for (int rl0 = warp; rl0 < RG * 16; rl0 += kNWC * RB) {
    int rr_[RB];
    float val[RB][NV], lse2[RB];
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      const int rl = rl0 + k * kNWC;
      const int r = rt * a.row_tile + rl;
      rr_[k] = (rl < RG * 16 && r < Rb) ? r : -1;
      const int rgi = (rl >> 4) < RG ? (rl >> 4) : RG - 1, rr = rl & 15;
      float M = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) M = fmaxf(M, redM[(rgi + kk * RG) * 16 + rr]);
      const float bse = (M == -INFINITY) ? 0.f : M;
      float lsum = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j) val[k][j] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int wi = rgi + kk * RG;
        const float w = fast_exp2(redM[wi * 16 + rr] - bse);
        lsum += w * redL[wi * 16 + rr];
        const float* src = &redO[(wi * 16 + rr) * S::kRedStride + lane * NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) val[k][j] += w * src[j];
      }
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j) val[k][j] *= inv;
      lse2[k] = lsum > 0.f ? bse + log2f(lsum) : -INFINITY;
    }
    if (a.n_splits > 1) {
#pragma unroll
      for (int k = 0; k < RB; ++k)
        if (rr_[k] >= 0) store_row<NV>(a, b, hk, split, rr_[k], val[k], lane * NV, 1, lse2[k], lane == 0);
    } else {
      write_final_rows<NV, RB>(a, b, hk, rr_, val, lse2, lane);
    }
  }
}

// ---------------------------------------------------------------------------
// fp32 CUDA-core kernel: row tile 16 (4 warps x 4 rows), tiles of kTK keys.
// A tile's K and V arrive by cp.async in one round trip into a two-stage ring
// (the next tile loads while this one is computed); K rows are padded to
// D + 4 floats so that lanes reading float4s of different keys hit different
// banks. Lane j of a warp owns keys j and j + 32 of the tile; the warp's 4 rows
// share every K load. P goes through shared memory for the PV product.
// ---------------------------------------------------------------------------
constexpr int kF32Rows = 16;

template <int D>
struct F32Smem {
  static constexpr int KP = D + 4;
  static constexpr int bytes =
      4 * (kF32Rows * D + 2 * kTK * KP + 2 * kTK * D + kF32Rows * kTK);  // Q, K, V, P
};

template <int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const __grid_constant__ AttnArgs a) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  constexpr int NV = D / 32, KP = F32Smem<D>::KP, C4 = D / 4;
  extern __shared__ __align__(16) float fs[];
  float* Qs = fs;                   // [kF32Rows][D]
  float* Ks = Qs + kF32Rows * D;    // [2][kTK][KP]
  float* Vs = Ks + 2 * kTK * KP;    // [2][kTK][D]
  float* Ps = Vs + 2 * kTK * D;     // [kF32Rows][kTK]
  __shared__ long long slots[2][kMaxChunks];
  __shared__ int meta[2][kMaxChunks];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x % a.n_row_tiles;
  const int split = blockIdx.x / a.n_row_tiles;
  const int hk = blockIdx.y, b = blockIdx.z;
  if (!cta_selected(a, b, hk)) return;
  const int Rb = rows_of(a, b);  // stacked rows of this sequence
  if (rt * a.row_tile >= Rb) return;
  const GroupInfo gi = group_info(a, b, hk);
  const int n_tiles = n_tiles_of(a, gi);
  const int tps = split_tiles(a, n_tiles, false);
  const int tile0 = split * tps;
  const int n_it = max(0, min(tps, n_tiles - tile0));
  const int n_chunks = kTK / a.chunk;
  const float* qf = static_cast<const float*>(a.q);
  const float* kg = static_cast<const float*>(a.k);
  const float* vg = static_cast<const float*>(a.v);

  for (int idx = tid; idx < kF32Rows * C4; idx += blockDim.x) {
    const int rl = idx / C4, c4 = idx - rl * C4;
    const int r = rt * kF32Rows + rl;
    if (r < Rb) {
      int i, h;
      row_of(a, b, hk, r, i, h);
      cp_async16(smem_u32(Qs + rl * D + 4 * c4), qf + ((q_row0(a, b) + i) * a.Hq + h) * D + 4 * c4,
                 16u);
    } else {
      *reinterpret_cast<float4*>(Qs + rl * D + 4 * c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  cp_async_commit();

  auto fill_meta = [&](int it, int st) {
    if (tid < n_chunks) {
      long long sl;
      int v;
      chunk_slot(a, gi, b, hk, tile0 + it, tid, sl, v);
      slots[st][tid] = sl;
      meta[st][tid] = v;
    }
  };
  // keys outside the key set are zero-filled (and masked below)
  auto issue = [&](int st) {
    for (int idx = tid; idx < kTK * C4; idx += blockDim.x) {
      const int key = idx / C4, c4 = idx - key * C4;
      const int ci = key / a.chunk, off = key - ci * a.chunk;
      const bool ok = off < meta[st][ci];
      const long long e = ok ? ((slots[st][ci] + off) * a.Hkv + hk) * D + 4 * c4 : 0;
      cp_async16(smem_u32(Ks + (st * kTK + key) * KP + 4 * c4), kg + e, ok ? 16u : 0u);
      cp_async16(smem_u32(Vs + (st * kTK + key) * D + 4 * c4), vg + e, ok ? 16u : 0u);
    }
    cp_async_commit();
  };

  float m_r[4], l_r[4], o[4][NV];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    m_r[k] = -INFINITY;
    l_r[k] = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) o[k][j] = 0.f;
  }

  if (n_it > 0) {
    fill_meta(0, 0);
    __syncthreads();
    issue(0);
  }
  for (int it = 0; it < n_it; ++it) {
    const int st = it & 1;
    if (it + 1 < n_it) {
      fill_meta(it + 1, st ^ 1);
      __syncthreads();
      issue(st ^ 1);
      cp_async_wait<1>();  // Q and this tile have landed
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* K = Ks + st * kTK * KP;
    const float* V = Vs + st * kTK * D;
    bool valid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int key = lane + 32 * h, ci = key / a.chunk;
      valid[h] = key - ci * a.chunk < meta[st][ci];
    }
    float s[4][2];
#pragma unroll
    for (int k = 0; k < 4; ++k) s[k][0] = s[k][1] = 0.f;
#pragma unroll 4
    for (int c4 = 0; c4 < C4; ++c4) {
      const float4 k0 = *reinterpret_cast<const float4*>(K + lane * KP + 4 * c4);
      const float4 k1 = *reinterpret_cast<const float4*>(K + (lane + 32) * KP + 4 * c4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 q = *reinterpret_cast<const float4*>(Qs + (warp * 4 + k) * D + 4 * c4);
        s[k][0] = fmaf(q.x, k0.x, fmaf(q.y, k0.y, fmaf(q.z, k0.z, fmaf(q.w, k0.w, s[k][0]))));
        s[k][1] = fmaf(q.x, k1.x, fmaf(q.y, k1.y, fmaf(q.z, k1.z, fmaf(q.w, k1.w, s[k][1]))));
      }
    }
    float* P = Ps + warp * 4 * kTK;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float s0 = valid[0] ? s[k][0] * a.scale_log2 : -INFINITY;
      const float s1 = valid[1] ? s[k][1] * a.scale_log2 : -INFINITY;
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m_r[k], mx);
      const float bse = (mn == -INFINITY) ? 0.f : mn;
      const float alpha = exp2f(m_r[k] - bse);
      const float p0 = exp2f(s0 - bse), p1 = exp2f(s1 - bse);
      float ps = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_r[k] = l_r[k] * alpha + ps;
      m_r[k] = mn;
#pragma unroll
      for (int j = 0; j < NV; ++j) o[k][j] *= alpha;
      P[k * kTK + lane] = p0;
      P[k * kTK + lane + 32] = p1;
    }
    __syncwarp();
#pragma unroll 2
    for (int jk = 0; jk < kTK; jk += 4) {
      float4 pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) pk[k] = *reinterpret_cast<const float4*>(P + k * kTK + jk);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const float vv = V[(jk + u) * D + lane + 32 * j];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float pu = u == 0 ? pk[k].x : (u == 1 ? pk[k].y : (u == 2 ? pk[k].z : pk[k].w));
            o[k][j] = fmaf(pu, vv, o[k][j]);
          }
        }
      }
    }
    __syncthreads();  // stage st, its meta and P are free for the next prefetch
  }
  if (n_it == 0) cp_async_wait<0>();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = rt * kF32Rows + warp * 4 + k;
    if (r >= Rb) break;
    const float inv = l_r[k] > 0.f ? 1.f / l_r[k] : 0.f;
    float val[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) val[j] = o[k][j] * inv;
    const float lse2 = l_r[k] > 0.f ? m_r[k] + log2f(l_r[k]) : -INFINITY;
    store_row<NV>(a, b, hk, split, r, val, lane, 32, lse2, lane == 0);
  }
}

// ---------------------------------------------------------------------------
// Split-KV combine: one warp per row of (b, hk); same log-space rule as the
// FlashBlock merge, over n_splits partials (an empty split has weight 0 and
// is left out of the sum).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ AttnArgs a) {
  // Launched as a programmatic dependent of the partial kernel: wait until that
  // grid has completed and its partials are visible (no-op on a plain launch).
  grid_dependency_wait();
  allow_dependent_launch();
  constexpr int NV = D / 32;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)a.batch * a.Hkv * a.R;
  if (warp >= rows) return;
  const int r = warp % a.R;
  const int hk = (warp / a.R) % a.Hkv;
  const int b = warp / (a.R * a.Hkv);
  if (r >= rows_of(a, b)) return;  // packed rows: past this sequence's count
  int i, h;
  row_of(a, b, hk, r, i, h);
  if (!row_selected(a, b, h)) return;
  combine_row<NV>(a, b, hk, r, lane);
}

// ---------------------------------------------------------------------------
// FlashBlock merge (technical summary §2, merge equation), one warp per row:
//   m = max(L_out, L_in), w_x = e^{L_x - m},
//   A_full = (w_out A_out + w_in A_in) / (w_out + w_in), L_full = m + log(w_out + w_in)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    merge_kernel(const float* __restrict__ a_out, const float* __restrict__ l_out,
                 const float* __restrict__ a_in, const float* __restrict__ l_in, long long rows,
                 float* __restrict__ a_full, float* __restrict__ l_full) {
  constexpr int NV = D / 32;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float lo = l_out[warp], li = l_in[warp];
  const float m = fmaxf(lo, li);
  float wo = 0.f, wi = 0.f, den = 1.f, L = -INFINITY;
  if (m != -INFINITY) {
    wo = expf(lo - m);
    wi = expf(li - m);
    den = wo + wi;
    L = m + logf(den);
  }
  const float inv = 1.f / den;
  const float* so = a_out + warp * D + lane * NV;
  const float* si = a_in + warp * D + lane * NV;
  float* dst = a_full + warp * D + lane * NV;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    // a side whose weight is 0 is not read (it may hold stale bits)
    const float x = (wo > 0.f ? wo * so[j] : 0.f) + (wi > 0.f ? wi * si[j] : 0.f);
    dst[j] = x * inv;
  }
  if (l_full && lane == 0) l_full[warp] = L;
}

}  // namespace fb
