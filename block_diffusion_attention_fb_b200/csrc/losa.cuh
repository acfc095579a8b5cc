// LoSA selection kernels ("LoSA: Locality Aware Sparse Attention for
// Block-Wise Diffusion Language Models", §2 "El Algoritmo LoSA", steps 1 and 3)
// and the per-page key summaries its QUEST-style selector scores.
//
// Decisions are integers chosen by float scores, so every score is computed
// in one fixed float32 order: single-rounded products (__fmul_rn), and sums by
// the stride-halving tree (pad to a power of two N; for stride = N/2 ... 1,
// x[n] += x[n + stride] for n < stride). Ties go to the lower index.
#pragma once

#include "common.cuh"

namespace fb {

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);  // exact here: x is a bf16 value
}

struct KvView {
  const void* k;
  const int32_t* page_table;
  const int32_t* seq_len;
  long long n_slots;
  int batch, Hkv, D, page_size, max_pages, max_seq_len;
};

__device__ __forceinline__ int kv_tokens(const KvView& kv, int b) {
  return kv.seq_len ? kv.seq_len[b] : kv.max_seq_len;
}

// Pool row of token t of sequence b, or -1 when the page-table entry lies
// outside the pool (the error word then records it; no access is made).
__device__ __forceinline__ long long kv_slot(const KvView& kv, int b, int t) {
  if (kv.page_table) {
    const int lp = t / kv.page_size;
    const int pg = kv.page_table[(long long)b * kv.max_pages + lp];
    if (pg < 0 || ((long long)pg + 1) * kv.page_size > kv.n_slots) {
      atomicOr(&g_fb_error_word, kErrBadReadPage);
      return -1;
    }
    return (long long)pg * kv.page_size + (t - lp * kv.page_size);
  }
  return (long long)b * kv.max_seq_len + t;
}

// ---------------------------------------------------------------------------
// Per (sequence, logical page, kv head, channel): min and max of the page's
// valid keys. One warp per (b, page, hk); lanes hold channels lane + 32 j.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
    page_summary_kernel(const KvView kv, T* __restrict__ pmin, T* __restrict__ pmax) {
  constexpr int NV = D / 32;
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)kv.batch * kv.max_pages * kv.Hkv;
  if (w >= total) return;
  const int hk = (int)(w % kv.Hkv);
  const int p = (int)((w / kv.Hkv) % kv.max_pages);
  const int b = (int)(w / ((long long)kv.Hkv * kv.max_pages));
  const int n = kv_tokens(kv, b);
  const int t0 = p * kv.page_size;
  if (t0 >= n) return;
  const int t1 = min(n, t0 + kv.page_size);
  const T* kg = static_cast<const T*>(kv.k);
  float mn[NV], mx[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    mn[j] = INFINITY;
    mx[j] = -INFINITY;
  }
  for (int t = t0; t < t1; ++t) {
    const long long slot = kv_slot(kv, b, t);
    if (slot < 0) continue;
    const T* row = kg + (slot * kv.Hkv + hk) * D;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const float x = ld_f32<T>(row + lane + 32 * j);
      mn[j] = fminf(mn[j], x);
      mx[j] = fmaxf(mx[j], x);
    }
  }
  const long long o = (((long long)b * kv.max_pages + p) * kv.Hkv + hk) * D;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    pmin[o + lane + 32 * j] = from_f32<T>(mn[j]);
    pmax[o + lane + 32 * j] = from_f32<T>(mx[j]);
  }
}

// ---------------------------------------------------------------------------
// Step 1a: locality score of every block row, sum_{h,c} (q_cur - q_prev)^2
// by the stride-halving tree over n = h * D + c. One CTA per (row, sequence);
// the tree runs level by level in shared memory exactly as defined.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
    locality_score_kernel(const T* __restrict__ qc, const T* __restrict__ qp, int B, int N,
                          int N2, float* __restrict__ score) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  extern __shared__ float xs[];  // N2 floats
  const int i = blockIdx.x, b = blockIdx.y;
  const long long off = ((long long)b * B + i) * N;
  for (int n = threadIdx.x; n < N2; n += blockDim.x) {
    float v = 0.f;
    if (n < N) {
      const float d = __fsub_rn(ld_f32<T>(qc + off + n), ld_f32<T>(qp + off + n));
      v = __fmul_rn(d, d);
    }
    xs[n] = v;
  }
  __syncthreads();
  for (int s = N2 >> 1; s >= 1; s >>= 1) {
    for (int n = threadIdx.x; n < s; n += blockDim.x) xs[n] = __fadd_rn(xs[n], xs[n + s]);
    __syncthreads();
  }
  if (threadIdx.x == 0) score[(long long)b * B + i] = xs[0];
}

// Same score with the tree in registers: 256 threads, thread t owns elements
// n = t + 256 j (j < E, E = N2 / 256), so the tree levels with stride >= 256
// pair j with j + E/2, ... inside the thread; strides 128..32 go through
// shared memory and 16..1 through xor shuffles (lane t + s for t < s).
template <typename T, int E>
__global__ void __launch_bounds__(256)
    locality_score_reg_kernel(const T* __restrict__ qc, const T* __restrict__ qp, int B, int N,
                              float* __restrict__ score) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  __shared__ float red[256];
  const int i = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const long long off = ((long long)b * B + i) * N;
  float x[E];
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const int n = t + 256 * j;
    float v = 0.f;
    if (n < N) {
      const float d = __fsub_rn(ld_f32<T>(qc + off + n), ld_f32<T>(qp + off + n));
      v = __fmul_rn(d, d);
    }
    x[j] = v;
  }
#pragma unroll
  for (int s = E / 2; s >= 1; s >>= 1)
#pragma unroll
    for (int j = 0; j < s; ++j) x[j] = __fadd_rn(x[j], x[j + s]);
  red[t] = x[0];
  __syncthreads();
#pragma unroll
  for (int s = 128; s >= 32; s >>= 1) {
    if (t < s) red[t] = __fadd_rn(red[t], red[t + s]);
    __syncthreads();
  }
  if (t < 32) {
    float v = red[t];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, s));
    if (t == 0) score[(long long)b * B + i] = v;
  }
}

// Step 1b: the n_act highest-scoring rows of each sequence, in rank order
// (score descending, then row ascending). Up to 32 active rows: n_act rounds
// of a block-wide maximum over the key (order-preserving score bits, ~row), so
// a higher score wins and equal scores go to the lower row; more active rows:
// O(B^2) ranks. Scores are sums of squares, never NaN.
//
// The rounds, for one sequence, by the whole CTA (blockDim a multiple of 32,
// at most 1024): score_b [B] from global, sc [B] shared scratch, taken [32]
// receives the rows in rank order (shared). Every thread returns after the
// last round's barrier, so taken[] is visible to all.
__device__ __forceinline__ void pick_active_rows(const float* score_b, int B, int n_act,
                                                 float* sc, int* taken) {
  __shared__ unsigned long long wbest[32];
  for (int i0 = threadIdx.x; i0 < B; i0 += 8 * blockDim.x) {  // 8 loads in flight
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      v[u] = i < B ? __ldcg(score_b + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < B) sc[i] = v[u];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int r = 0; r < n_act; ++r) {
    unsigned long long best = 0ull;
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
      bool used = false;
      for (int t = 0; t < r; ++t) used |= (taken[t] == i);
      if (used) continue;
      const float f = sc[i] == 0.f ? 0.f : sc[i];  // -0 and +0 rank equal
      const uint32_t u = __float_as_uint(f);
      const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      const unsigned long long k = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
      best = k > best ? k : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (lane == 0) wbest[wid] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long m = 0ull;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = wbest[w] > m ? wbest[w] : m;
      taken[r] = (int)(0xFFFFFFFFu - (uint32_t)(m & 0xFFFFFFFFull));
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256)
    active_rows_kernel(const float* __restrict__ score, int B, int n_act,
                       int32_t* __restrict__ active) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  extern __shared__ float sc[];
  const int b = blockIdx.x;
  if (n_act <= 32) {
    __shared__ int taken[32];
    pick_active_rows(score + (long long)b * B, B, n_act, sc, taken);
    for (int r = threadIdx.x; r < n_act; r += blockDim.x) active[b * n_act + r] = taken[r];
    return;
  }
  for (int i = threadIdx.x; i < B; i += blockDim.x) sc[i] = score[(long long)b * B + i];
  __syncthreads();
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const float si = sc[i];
    int rank = 0;
    for (int j = 0; j < B; ++j) {
      const float sj = sc[j];
      rank += (sj > si) || (sj == si && j < i);
    }
    if (rank < n_act) active[b * n_act + rank] = i;
  }
}

// ---------------------------------------------------------------------------
// Page scoring (steps 3a of LoSA and the sparse-residual selector): pages are
// handled in chunks of kPsPages.
// ---------------------------------------------------------------------------
constexpr int kPsPages = 64;
// chunk buffers of the page scorers: bf16 three (two load while one is scored),
// float32 two (its chunks are twice as large)
__host__ __device__ constexpr int ps_stages(int elem_bytes) { return elem_bytes == 2 ? 3 : 2; }

// Shared-memory row stride (elements) of the staged page summaries: rows stay
// 16-byte aligned for vector loads, and consecutive pages start 4 banks apart,
// so the 8 lanes of a quarter warp reading 16 bytes each hit distinct banks.
template <typename T, int D>
__host__ __device__ constexpr int ps_stride() {
  return D + 16 / (int)sizeof(T);
}

// 8 consecutive elements as float (exact for bf16 and f32) from shared memory.
__device__ __forceinline__ void load8_f32(const __nv_bfloat16* p, float (&o)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[2 * j] = __uint_as_float(w[j] << 16);
    o[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8_f32(const float* p, float (&o)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

// QUEST-style bound of one q row over one staged page:
//   tree_sum_c max(q_c * kmin_c, q_c * kmax_c)
// single-rounded products, then the stride-halving tree over c (level 1 pairs
// c with c + D/2). Operands are read 8 channels per shared-memory load; the
// arithmetic and its order are those of the definition.
template <typename T, int D>
__device__ __forceinline__ float page_bound(const float* qr, const T* mnr, const T* mxr) {
  float y[D / 2];
#pragma unroll
  for (int c8 = 0; c8 < D / 2; c8 += 8) {
    float q0[8], q1[8], n0[8], n1[8], x0[8], x1[8];
    load8_f32(qr + c8, q0);
    load8_f32(qr + c8 + D / 2, q1);
    load8_f32(mnr + c8, n0);
    load8_f32(mnr + c8 + D / 2, n1);
    load8_f32(mxr + c8, x0);
    load8_f32(mxr + c8 + D / 2, x1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float a0 = fmaxf(__fmul_rn(q0[j], n0[j]), __fmul_rn(q0[j], x0[j]));
      const float a1 = fmaxf(__fmul_rn(q1[j], n1[j]), __fmul_rn(q1[j], x1[j]));
      y[c8 + j] = __fadd_rn(a0, a1);
    }
  }
#pragma unroll
  for (int st = D / 4; st >= 1; st >>= 1)
#pragma unroll
    for (int c = 0; c < st; ++c) y[c] = __fadd_rn(y[c], y[c + st]);
  return y[0];
}

// The same bound for bf16 inputs, evaluated as tree_sum_c q_c * s_c with s_c =
// kmax_c where q_c >= 0 and kmin_c where q_c < 0. A product of two bf16 values
// is exact in float32, so max(q_c kmin_c, q_c kmax_c) IS q_c s_c, bit for bit
// (for q_c = 0 both are zeros); the products and the tree are unchanged, only
// the selection happens before the multiply. Two channels per 32-bit word: the
// per-row mask qm (0xFFFF in the half of each channel with q_c < 0) picks the
// bf16 halves with one bitwise select; products and tree levels with stride >= 2
// run on packed float pairs (f32x2), each lane single-rounded as in the
// definition. q row qr (float) and qm are read by every lane of the warp at the
// same address (broadcast); mnr / mxr are this lane's page.
template <int D>
__device__ __forceinline__ float page_bound_sel(const float* qr, const uint32_t* qm,
                                                const __nv_bfloat16* mnr,
                                                const __nv_bfloat16* mxr) {
  // The first three tree levels (channel strides D/2, D/4, D/8) are formed per
  // output channel n < E = D/8 from the eight channels n + k E, k = 0..7:
  //   ((a_n + a_n+4E) + (a_n+2E + a_n+6E)) + ((a_n+E + a_n+5E) + (a_n+3E + a_n+7E)),
  // which is the tree's own pairing and order; only E values stay live.
  constexpr int E = D / 8;
  float2 z[E / 2];  // level-3 sums of channels (2i, 2i + 1)
  // products of the channel pairs c8 + 2j (+1) + k E, j = 0..3
  auto prod = [&](int c8, int k, float2 (&a)[4]) {
    const int c = c8 + k * E;
    const uint4 n = *reinterpret_cast<const uint4*>(mnr + c);
    const uint4 x = *reinterpret_cast<const uint4*>(mxr + c);
    const uint4 m = *reinterpret_cast<const uint4*>(qm + c / 2);
    const float4 qa = *reinterpret_cast<const float4*>(qr + c);
    const float4 qb = *reinterpret_cast<const float4*>(qr + c + 4);
    const uint32_t nn[4] = {n.x, n.y, n.z, n.w}, xx[4] = {x.x, x.y, x.z, x.w};
    const uint32_t mm[4] = {m.x, m.y, m.z, m.w};
    const float2 qq[4] = {make_float2(qa.x, qa.y), make_float2(qa.z, qa.w),
                          make_float2(qb.x, qb.y), make_float2(qb.z, qb.w)};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t sel = (xx[j] & ~mm[j]) | (nn[j] & mm[j]);
      a[j] = fmul2(qq[j], make_float2(__uint_as_float(sel << 16),
                                      __uint_as_float(sel & 0xFFFF0000u)));
    }
  };
  // level-1 pair (k, k + 4) of the eight offsets
  auto level1 = [&](int c8, int k, float2 (&b)[4]) {
    float2 lo[4], hi[4];
    prod(c8, k, lo);
    prod(c8, k + 4, hi);
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = fadd2(lo[j], hi[j]);
  };
#pragma unroll
  for (int c8 = 0; c8 < E; c8 += 8) {
    // keeps the next group's loads from being hoisted above this one (which
    // would hold both groups' operands at once and spill)
    if (c8 > 0) asm volatile("" ::: "memory");
    float2 b0[4], b2[4], c0[4];
    level1(c8, 0, b0);
    level1(c8, 2, b2);
#pragma unroll
    for (int j = 0; j < 4; ++j) c0[j] = fadd2(b0[j], b2[j]);
    float2 b1[4], b3[4];
    level1(c8, 1, b1);
    level1(c8, 3, b3);
#pragma unroll
    for (int j = 0; j < 4; ++j) z[c8 / 2 + j] = fadd2(c0[j], fadd2(b1[j], b3[j]));
  }
#pragma unroll
  for (int st = E / 4; st >= 1; st >>= 1)  // channel strides 2 st = E/2 ... 2, in pairs
#pragma unroll
    for (int i = 0; i < st; ++i) z[i] = fadd2(z[i], z[i + st]);
  return __fadd_rn(z[0].x, z[0].y);  // the last level: channel 0 + channel 1
}

// Shared memory of the page scorers for RQ staged q rows: the rows (float),
// their sign masks (bf16 inputs), and two buffers of a chunk's summaries.
__host__ __device__ constexpr int page_score_smem(int RQ, int D, int elem_bytes) {
  return RQ * D * 4 + (elem_bytes == 2 ? RQ * (D / 2) * 4 : 0) +
         2 * ps_stages(elem_bytes) * kPsPages * (D + 16 / elem_bytes) * elem_bytes;
}

// Stages the active q rows of (b, hk) as float, and for bf16 the per-channel
// sign masks of page_bound_sel: qs [RQ][D], qm [RQ][D/2].
// act: the n_act active rows of sequence b (global or shared), or NULL for
// rows 0 .. n_act-1. Stacked rows row0 .. row0 + RQ - 1 are staged.
template <typename T, int D>
__device__ __forceinline__ void stage_q_rows(const T* q, const int* act, int b, int B,
                                             int Hq, int G, int hk, int n_act, int RQ, float* qs,
                                             uint32_t* qm, int row0 = 0) {
  for (int idx = threadIdx.x; idx < RQ * D; idx += blockDim.x) {
    const int rq = idx / D, c = idx - (idx / D) * D;
    const int a_i = (row0 + rq) / G, g = (row0 + rq) - a_i * G;
    const int i = act ? act[a_i] : a_i;
    qs[idx] = ld_f32<T>(q + (((long long)b * B + i) * Hq + hk * G + g) * D + c);
  }
  if constexpr (sizeof(T) == 2) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < RQ * (D / 2); idx += blockDim.x) {
      const int rq = idx / (D / 2), c2 = idx - rq * (D / 2);
      const uint32_t lo = __float_as_uint(qs[rq * D + 2 * c2]) >> 31;
      const uint32_t hi = __float_as_uint(qs[rq * D + 2 * c2 + 1]) >> 31;
      qm[idx] = (lo ? 0x0000FFFFu : 0u) | (hi ? 0xFFFF0000u : 0u);
    }
  }
}

// Stages the summaries of 64-page chunk `chunk` of (b, hk) into one of two
// shared buffers with cp.async (zero-filled past the sequence's pages).
template <typename T, int D>
__device__ __forceinline__ void stage_page_chunk(const T* pmin, const T* pmax, const KvView& kv,
                                                 int b, int hk, int chunk, int n_pages,
                                                 T* smn, T* smx) {
  constexpr int PS = ps_stride<T, D>();
  constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte copy
  for (int idx = threadIdx.x; idx < kPsPages * (D / VE); idx += blockDim.x) {
    const int pg = idx / (D / VE), cv = idx - (idx / (D / VE)) * (D / VE);
    const int p = chunk * kPsPages + pg;
    const bool ok = p < n_pages;
    const long long so = (((long long)b * kv.max_pages + (ok ? p : 0)) * kv.Hkv + hk) * D + cv * VE;
    cp_async16(smem_u32(smn + pg * PS + cv * VE), pmin + so, ok ? 16u : 0u);
    cp_async16(smem_u32(smx + pg * PS + cv * VE), pmax + so, ok ? 16u : 0u);
  }
}

// The chunk ring of the page scorers: chunks c0 .. c1-1 of (b, hk) cycle
// through kStages buffers of [64][PS] minima then [64][PS] maxima. One
// cp.async group is committed per chunk (empty past c1), so that waiting for
// all but the newest kStages - 1 groups means chunk ch has landed.
template <typename T, int D>
struct PageRing {
  T* sbuf;
  const T* pmin;
  const T* pmax;
  const KvView& kv;
  int b, hk, c0, c1, n_pages;
  static constexpr int PS = ps_stride<T, D>();
  static constexpr int kStages = ps_stages((int)sizeof(T));
  __device__ T* mn(int ch) const { return sbuf + ((ch - c0) % kStages) * 2 * kPsPages * PS; }
  __device__ T* mx(int ch) const { return mn(ch) + kPsPages * PS; }
  __device__ void issue(int ch) const {
    if (ch < c1) stage_page_chunk<T, D>(pmin, pmax, kv, b, hk, ch, n_pages, mn(ch), mx(ch));
    cp_async_commit();
  }
  __device__ void prologue() const {
#pragma unroll
    for (int k = 0; k < kStages - 1; ++k) issue(c0 + k);
  }
  // before scoring chunk ch: load chunk ch + kStages - 1 into the buffer that
  // chunk ch - 1 left (the caller's trailing __syncthreads freed it), wait for ch
  __device__ void advance(int ch) const {
    issue(ch + kStages - 1);
    cp_async_wait<kStages - 1>();
  }
};

// Step 3a: QUEST-style page scores u_p = tree_sum_c max(q_c kmin_c, q_c kmax_c)
// for every active row a and q head h of kv head hk. A CTA scores `cpc`
// consecutive chunks of 64 pages of one (b, hk): the active q rows once into
// shared memory, the summaries chunk by chunk into two buffers with cp.async,
// the next chunk loading while the current one is scored. bf16: a warp takes
// one q row (broadcast reads) and 32 pages (one per lane; warps 2r and 2r+1
// the two halves of the chunk, rows r, r + 4, ... for the 8 warps), bound by
// page_bound_sel; float32: one thread per (page, row) by page_bound. Both are
// single-rounded products and the stride-halving tree.
// scores: [batch, n_act, Hq, max_pages]. Block (0, hk, b) also clears the
// union bitmap of (b, hk) and its ticket for the top-k kernel that follows.
// Active rows: given (active), or picked here from the locality scores
// row_scores [batch, B] (n_act <= 32; every CTA of a sequence picks the same
// rows, block (0, 0, b) writes them to active_out).
template <typename T, int D>
__global__ void __launch_bounds__(256, 2)
    page_score_kernel(const T* __restrict__ q, const int32_t* __restrict__ active,
                      const float* __restrict__ row_scores, int32_t* __restrict__ active_out,
                      int B, int Hq, int G, int n_act, const T* __restrict__ pmin,
                      const T* __restrict__ pmax, const KvView kv, float* __restrict__ scores,
                      uint32_t* __restrict__ bitmap, int words, int* __restrict__ tickets,
                      int cpc) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  constexpr int PS = ps_stride<T, D>();
  constexpr bool kSel = sizeof(T) == 2;  // bf16: masked-select bound, warp per row
  extern __shared__ __align__(16) float sm[];
  __shared__ int s_active[32];
  const int RQ = n_act * G;
  float* qs = sm;                                            // [RQ][D]
  uint32_t* qm = reinterpret_cast<uint32_t*>(qs + RQ * D);   // [RQ][D/2] (bf16)
  T* sbuf = reinterpret_cast<T*>(qm + (kSel ? RQ * (D / 2) : 0));  // stages of [64][PS] min, max
  float* sc = reinterpret_cast<float*>(sbuf + 2 * ps_stages((int)sizeof(T)) * kPsPages * PS);
  const int hk = blockIdx.y, b = blockIdx.z;
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < words; w += blockDim.x)
      bitmap[((long long)b * kv.Hkv + hk) * words + w] = 0u;
    if (tickets && threadIdx.x == 0) tickets[b * kv.Hkv + hk] = 0;
  }
  const int n_pages = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const int c0 = blockIdx.x * cpc;
  const int c1 = min(c0 + cpc, (n_pages + kPsPages - 1) / kPsPages);
  const bool pick = row_scores != nullptr;
  if (c0 >= c1 && !(pick && blockIdx.x == 0 && hk == 0)) return;
  const int* act = active ? active + b * n_act : nullptr;
  if (pick) {
    pick_active_rows(row_scores + (long long)b * B, B, n_act, sc, s_active);
    if (blockIdx.x == 0 && hk == 0)
      for (int r = threadIdx.x; r < n_act; r += blockDim.x) active_out[b * n_act + r] = s_active[r];
    if (c0 >= c1) return;
    act = s_active;
  }
  const PageRing<T, D> ring{sbuf, pmin, pmax, kv, b, hk, c0, c1, n_pages};
  ring.prologue();
  stage_q_rows<T, D>(q, act, b, B, Hq, G, hk, n_act, RQ, qs, qm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, n_warps = blockDim.x >> 5;
  for (int ch = c0; ch < c1; ++ch) {
    ring.advance(ch);
    const T* smn = ring.mn(ch);
    const T* smx = ring.mx(ch);
    __syncthreads();  // chunk ch (and the q rows) visible to every thread
    if constexpr (kSel) {
      const int pg = (warp & 1) * 32 + lane;
      const int p = ch * kPsPages + pg;
      for (int rq = warp >> 1; rq < RQ; rq += n_warps >> 1) {
        const float yb = page_bound_sel<D>(qs + rq * D, qm + rq * (D / 2), smn + pg * PS,
                                           smx + pg * PS);
        const int a_i = rq / G, g = rq - (rq / G) * G;
        if (p < n_pages)
          scores[(((long long)b * n_act + a_i) * Hq + hk * G + g) * kv.max_pages + p] = yb;
      }
    } else {
      for (int task = threadIdx.x; task < kPsPages * RQ; task += blockDim.x) {
        const int pg = task % kPsPages, rq = task / kPsPages;
        const int p = ch * kPsPages + pg;
        if (p >= n_pages) continue;
        const float yb = page_bound<T, D>(qs + rq * D, smn + pg * PS, smx + pg * PS);
        const int a_i = rq / G, g = rq - (rq / G) * G;
        scores[(((long long)b * n_act + a_i) * Hq + hk * G + g) * kv.max_pages + p] = yb;
      }
    }
    __syncthreads();  // this chunk's buffer is refilled in the next iteration
  }
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 == +0.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Step 3b: top-k pages of one (active row, q head): exact radix select of the
// k-th largest key (4 passes of 8 bits), then every key above it plus the
// lowest-index keys equal to it. The picks are gathered in a shared bitmap and
// OR-ed into the union bitmap of the kv head one word at a time. One CTA of
// kTopkThreads per (b, a, h).
// Step 3c: the last of the n_act * G CTAs of a (b, hk) to finish (a ticket
// that the page scorer zeroed) turns the union bitmap into the ascending page
// list and count.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 512;

// Exclusive prefix sum over the CTA (blockDim a multiple of 32, at most 1024)
// of one value per thread; total receives the sum. Ends with a barrier.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int w = lane < nw ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < nw) warp_sums[lane] = wi - w;
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  total = warp_sums[32];
  const int res = warp_sums[wid] + incl - x;
  __syncthreads();  // warp_sums may be reused by the caller
  return res;
}

// Bitmap (words, read through L2) -> ascending list of set bits and their count.
__device__ __forceinline__ void compact_bitmap(const uint32_t* bm, int words, int32_t* out,
                                               int32_t* count, int* warp_sums) {
  const int per = (words + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per, w1 = min(words, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(__ldcg(bm + w));
  int total;
  int pos = block_exclusive_scan(c, warp_sums, total);
  if (threadIdx.x == 0) *count = total;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = __ldcg(bm + w);
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      out[pos++] = w * 32 + bit;
    }
  }
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_pages_kernel(const float* __restrict__ scores, const KvView kv, int Hq, int G, int n_act,
                      int topk, uint32_t* __restrict__ bitmap, int words,
                      int32_t* __restrict__ list, int32_t* __restrict__ count, int list_stride,
                      int* __restrict__ tickets) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  extern __shared__ uint32_t keys[];  // max_pages keys, then a words-long bitmap
  __shared__ int hist[256];
  __shared__ int whist[kTopkThreads / 32][256];  // per-warp digit counts
  __shared__ int warp_sums[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need, s_last;
  const int ah = blockIdx.x, b = blockIdx.y;
  const int h = ah % Hq;
  const int hk = h / G;
  const int tid = threadIdx.x;
  const int n = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const int k = min(topk, n);
  uint32_t* sbm = keys + kv.max_pages;
  uint32_t* bm = bitmap + ((long long)b * kv.Hkv + hk) * words;
  const float* sc = scores + ((long long)b * n_act * Hq + ah) * kv.max_pages;
  for (int w = tid; w < words; w += blockDim.x) sbm[w] = 0u;
  auto take = [&](int p) { atomicOr(&sbm[p >> 5], 1u << (p & 31)); };
  if (k == n) {
    __syncthreads();
    for (int p = tid; p < n; p += blockDim.x) take(p);
  } else if (k > 0) {
    // the scores, 8 loads in flight per thread (a loop of single loads would
    // pay the memory latency once per key it reads)
    for (int p0 = tid; p0 < n; p0 += 8 * blockDim.x) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * blockDim.x;
        v[u] = p < n ? __ldcg(sc + p) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * blockDim.x;
        if (p < n) keys[p] = order_key(v[u]);
      }
    }
    if (tid == 0) {
      s_prefix = 0u;
      s_need = k;
    }
    uint32_t mask = 0u;
    const int wid = tid >> 5;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int d = tid; d < (kTopkThreads / 32) * 256; d += blockDim.x) (&whist[0][0])[d] = 0;
      __syncthreads();
      const uint32_t prefix = s_prefix;
      // Scores of one row are alike, so a few digits take most keys (all of
      // them share one in the first pass): each warp counts into its own
      // histogram, so only a warp's own lanes contend for a counter.
      for (int p = tid; p < n; p += blockDim.x) {
        const uint32_t key = keys[p];
        if ((key & mask) == prefix) atomicAdd(&whist[wid][(key >> shift) & 0xFFu], 1);
      }
      __syncthreads();
      for (int d = tid; d < 256; d += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kTopkThreads / 32; ++w) c += whist[w][d];
        hist[d] = c;
      }
      __syncthreads();
      if (tid < 32) {
        // buckets in descending order: lane l owns digits 255-8l ... 248-8l
        int cnt[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          cnt[j] = hist[255 - 8 * tid - j];
          tot += cnt[j];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        const int need = s_need;
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
        const int owner = __ffs(hit) - 1;  // first lane whose running count reaches need
        if (tid == owner) {
          int cum = incl - tot, sel = 0, rem = need;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (cum + cnt[j] >= need) {
              sel = 255 - 8 * tid - j;
              rem = need - cum;
              break;
            }
            cum += cnt[j];
          }
          s_prefix = prefix | ((uint32_t)sel << shift);
          s_need = rem;
        }
      }
      mask |= 0xFFu << shift;
      __syncthreads();
    }
    const uint32_t T = s_prefix;  // key of the k-th largest score
    const int need = s_need;      // how many keys equal to T are taken
    // every key above T; count the keys equal to it
    int eq = 0;
    for (int p = tid; p < n; p += blockDim.x) {
      const uint32_t key = keys[p];
      if (key > T) take(p);
      eq += key == T;
    }
    int n_eq;
    block_exclusive_scan(eq, warp_sums, n_eq);
    if (n_eq == need) {
      for (int p = tid; p < n; p += blockDim.x)
        if (keys[p] == T) take(p);
    } else {
      // more keys equal the k-th largest than are taken: the lowest indices,
      // from a scan over per-thread index segments (thread order = index order)
      const int seg = (n + blockDim.x - 1) / blockDim.x;
      const int p0 = tid * seg, p1 = min(n, p0 + seg);
      int cnt = 0;
      for (int p = p0; p < p1; ++p) cnt += (keys[p] == T);
      int tot;
      int eq_before = block_exclusive_scan(cnt, warp_sums, tot);
      for (int p = p0; p < p1; ++p) {
        if (keys[p] == T) {
          if (eq_before < need) take(p);
          ++eq_before;
        }
      }
    }
  }
  __syncthreads();
  for (int w = tid; w < words; w += blockDim.x)
    if (sbm[w]) atomicOr(&bm[w], sbm[w]);
  // the last CTA of the (b, hk) group compacts the union
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&tickets[b * kv.Hkv + hk], 1) == n_act * G - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  compact_bitmap(bm, words, list + ((long long)b * kv.Hkv + hk) * list_stride,
                 count + b * kv.Hkv + hk, warp_sums);
}

// ---------------------------------------------------------------------------
// FlashBlock + sparse attention (FlashBlock technical summary §2, compatibility
// with sparse attention): the sparse selector scores pages per kv head by the
// same QUEST-style bound, taking the maximum over every block row and every q
// head of the kv head: head score of page p = max_{i,g} tree_sum_c
// max(q_c kmin_c, q_c kmax_c). The per-(row, head) bound is formed exactly as in
// page_score_kernel (single-rounded products, stride-halving tree); the maximum
// is order-free, taken on order-preserving keys with shared-memory atomics.
// scores: [batch, Hkv, max_pages]. Block (0, hk, b) clears the (b, hk) bitmap.
// Rows are taken kHsRows at a time (q staged per group, every page chunk
// streamed again per group, from L2 where it fits): the maximum is order-free,
// and later groups fold theirs into the scores the earlier groups wrote.
// ---------------------------------------------------------------------------
constexpr int kHsRows = 64;

__device__ __forceinline__ float order_key_inv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 2)
    head_page_score_kernel(const T* __restrict__ q, int B, int Hq, int G,
                           const T* __restrict__ pmin, const T* __restrict__ pmax,
                           const KvView kv, float* __restrict__ scores,
                           uint32_t* __restrict__ bitmap, int words, int* __restrict__ tickets,
                           int cpc) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  constexpr int PS = ps_stride<T, D>();
  constexpr bool kSel = sizeof(T) == 2;  // bf16: masked-select bound, warp per row
  extern __shared__ __align__(16) float sm[];
  __shared__ uint32_t best[kPsPages];
  const int RQ_all = B * G;
  const int RQmax = RQ_all < kHsRows ? RQ_all : kHsRows;
  float* qs = sm;                                              // [RQmax][D], row r = i * G + g
  uint32_t* qm = reinterpret_cast<uint32_t*>(qs + RQmax * D);  // [RQmax][D/2] (bf16)
  T* sbuf = reinterpret_cast<T*>(qm + (kSel ? RQmax * (D / 2) : 0));  // stages of [64][PS]
  const int hk = blockIdx.y, b = blockIdx.z;
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < words; w += blockDim.x)
      bitmap[((long long)b * kv.Hkv + hk) * words + w] = 0u;
    if (tickets && threadIdx.x == 0) tickets[b * kv.Hkv + hk] = 0;
  }
  const int n_pages = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const int c0 = blockIdx.x * cpc;
  const int c1 = min(c0 + cpc, (n_pages + kPsPages - 1) / kPsPages);
  if (c0 >= c1) return;
  const PageRing<T, D> ring{sbuf, pmin, pmax, kv, b, hk, c0, c1, n_pages};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, n_warps = blockDim.x >> 5;
  for (int row0 = 0; row0 < RQ_all; row0 += kHsRows) {
  const int RQ = RQ_all - row0 < kHsRows ? RQ_all - row0 : kHsRows;
  ring.prologue();
  stage_q_rows<T, D>(q, nullptr, b, B, Hq, G, hk, B, RQ, qs, qm, row0);
  for (int ch = c0; ch < c1; ++ch) {
    for (int pg = threadIdx.x; pg < kPsPages; pg += blockDim.x) best[pg] = 0u;  // below every key
    ring.advance(ch);
    const T* smn = ring.mn(ch);
    const T* smx = ring.mx(ch);
    __syncthreads();  // chunk ch, the q rows and the cleared maxima visible to every thread
    if constexpr (kSel) {
      const int pg = (warp & 1) * 32 + lane;
      uint32_t mx = 0u;  // below every key
      for (int rq = warp >> 1; rq < RQ; rq += n_warps >> 1)
        mx = max(mx, order_key(page_bound_sel<D>(qs + rq * D, qm + rq * (D / 2), smn + pg * PS,
                                                  smx + pg * PS)));
      if (ch * kPsPages + pg < n_pages) atomicMax(&best[pg], mx);
    } else {
      for (int task = threadIdx.x; task < kPsPages * RQ; task += blockDim.x) {
        const int pg = task % kPsPages, rq = task / kPsPages;
        const int p = ch * kPsPages + pg;
        if (p >= n_pages) continue;
        const float yb = page_bound<T, D>(qs + rq * D, smn + pg * PS, smx + pg * PS);
        atomicMax(&best[pg], order_key(yb));
      }
    }
    __syncthreads();
    for (int pg = threadIdx.x; pg < kPsPages; pg += blockDim.x) {
      const int p = ch * kPsPages + pg;
      if (p < n_pages) {
        float* dst = scores + ((long long)b * kv.Hkv + hk) * kv.max_pages + p;
        // this CTA alone writes these pages: fold into an earlier group's maximum
        *dst = order_key_inv(row0 == 0 ? best[pg] : max(best[pg], order_key(*dst)));
      }
    }
    __syncthreads();  // maxima read out, this chunk's buffer free for the next iteration
  }
  }
}

// Complement of a selection bitmap within a sequence's pages: ascending list of
// the pages p < n_pages(b) whose bit is clear, and their count, per (b, hk).
__global__ void __launch_bounds__(256)
    complement_compact_kernel(const uint32_t* __restrict__ bitmap, int words, const KvView kv,
                              int stride, int32_t* __restrict__ list,
                              int32_t* __restrict__ count) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  __shared__ int wsum[256];
  const int hk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int n_pages = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const uint32_t* bm = bitmap + ((long long)b * kv.Hkv + hk) * words;
  int32_t* out = list + ((long long)b * kv.Hkv + hk) * stride;
  const int per = (words + 255) / 256;
  const int w0 = tid * per, w1 = min(words, w0 + per);
  auto clear_bits = [&](int w) -> uint32_t {
    const int lo = w * 32;
    if (lo >= n_pages) return 0u;
    const uint32_t valid = (n_pages - lo >= 32) ? 0xFFFFFFFFu : ((1u << (n_pages - lo)) - 1u);
    return ~bm[w] & valid;
  };
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(clear_bits(w));
  wsum[tid] = c;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int t = 0; t < 256; ++t) {
      const int x = wsum[t];
      wsum[t] = run;
      run += x;
    }
    count[b * kv.Hkv + hk] = run;
  }
  __syncthreads();
  int pos = wsum[tid];
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = clear_bits(w);
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      out[pos++] = w * 32 + bit;
    }
  }
}

}  // namespace fb
