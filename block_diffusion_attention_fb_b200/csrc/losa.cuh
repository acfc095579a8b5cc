// LoSA selection kernels ("LoSA: Locality Aware Sparse Attention for
// Block-Wise Diffusion Language Models", §2 "El Algoritmo LoSA", steps 1 and 3)
// and the per-page key summaries its QUEST-style selector scores.
//
// Decisions are integers chosen by float scores, so every score is computed
// in one fixed float32 order: single-rounded products (__fmul_rn), and sums by
// the stride-halving tree (pad to a power of two N; for stride = N/2 ... 1,
// x[n] += x[n + stride] for n < stride). Ties go to the lower index.
#pragma once

#include <type_traits>

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
// Page scoring (steps 3a of LoSA and the sparse-residual selector), float32
// summaries: pages are handled in chunks of kPsPages, staged in shared memory.
// (bf16 summaries: page_score_cols_kernel below.)
// ---------------------------------------------------------------------------
constexpr int kPsPages = 64;
constexpr int kPsStages = 2;  // chunk buffers: one loads while the other is scored

// Shared-memory row stride (elements) of the staged page summaries: rows stay
// 16-byte aligned for vector loads, and consecutive pages start 4 banks apart,
// so the 8 lanes of a quarter warp reading 16 bytes each hit distinct banks.
template <typename T, int D>
__host__ __device__ constexpr int ps_stride() {
  return D + 16 / (int)sizeof(T);
}

// 8 consecutive floats from shared memory.
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

// Shared memory of the page scorers for RQ staged q rows: the rows, and the
// chunk buffers of minima and maxima.
__host__ __device__ constexpr int page_score_smem(int RQ, int D) {
  return RQ * D * 4 + 2 * kPsStages * kPsPages * (D + 4) * 4;
}

// Stages the active q rows of (b, hk): qs [RQ][D].
// act: the n_act active rows of sequence b (global or shared), or NULL for
// rows 0 .. n_act-1. Stacked rows row0 .. row0 + RQ - 1 are staged.
template <typename T, int D>
__device__ __forceinline__ void stage_q_rows(const T* q, const int* act, int b, int B,
                                             int Hq, int G, int hk, int n_act, int RQ, float* qs,
                                             int row0 = 0) {
  for (int idx = threadIdx.x; idx < RQ * D; idx += blockDim.x) {
    const int rq = idx / D, c = idx - (idx / D) * D;
    const int a_i = (row0 + rq) / G, g = (row0 + rq) - a_i * G;
    const int i = act ? act[a_i] : a_i;
    qs[idx] = ld_f32<T>(q + (((long long)b * B + i) * Hq + hk * G + g) * D + c);
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
  static constexpr int kStages = kPsStages;
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
// the next chunk loading while the current one is scored; one thread per
// (page, row) by page_bound (single-rounded products, stride-halving tree).
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
  static_assert(sizeof(T) == 4, "float32 summaries (bf16: page_score_cols_kernel)");
  constexpr int PS = ps_stride<T, D>();
  extern __shared__ __align__(16) float sm[];
  __shared__ int s_active[32];
  const int RQ = n_act * G;
  float* qs = sm;                                    // [RQ][D]
  T* sbuf = reinterpret_cast<T*>(qs + RQ * D);       // stages of [64][PS] min, max
  float* sc = reinterpret_cast<float*>(sbuf + 2 * kPsStages * kPsPages * PS);
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
  stage_q_rows<T, D>(q, act, b, B, Hq, G, hk, n_act, RQ, qs);
  for (int ch = c0; ch < c1; ++ch) {
    ring.advance(ch);
    const T* smn = ring.mn(ch);
    const T* smx = ring.mx(ch);
    __syncthreads();  // chunk ch (and the q rows) visible to every thread
    for (int task = threadIdx.x; task < kPsPages * RQ; task += blockDim.x) {
      const int pg = task % kPsPages, rq = task / kPsPages;
      const int p = ch * kPsPages + pg;
      if (p >= n_pages) continue;
      const float yb = page_bound<T, D>(qs + rq * D, smn + pg * PS, smx + pg * PS);
      const int a_i = rq / G, g = rq - (rq / G) * G;
      scores[(((long long)b * n_act + a_i) * Hq + hk * G + g) * kv.max_pages + p] = yb;
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

__device__ __forceinline__ float order_key_inv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ---------------------------------------------------------------------------
// Step 3a, bf16 summaries: the same bounds with the lanes on channels. A warp
// scores a tile of kPcPages pages for kPcRows q rows at a time (32 bounds):
// lane l holds the channel pairs l + 32 k (channels 2l, 2l + 1, 2l + 64, ...),
// reads them for each page straight from global memory (a warp reads 128
// contiguous bytes per load), and forms each channel's bound as
//   fma(q-_c, kmin_c, q+_c * kmax_c),  q+ = max(q, 0), q- = min(q, 0),
// which is max(q_c kmin_c, q_c kmax_c) exactly: one of the two products is
// zero and the other is exact in fp32 (bf16 times bf16). The tree levels with
// channel stride >= 64 are lane-local; the lane's pair (2l, 2l + 1) of each of
// the 32 bounds then goes through a per-warp shared-memory transpose, and lane
// o finishes bound o: levels of stride 32 .. 2 pair v[i] with v[i + s/2], the
// last adds the pair's two channels. Every addition pairs the same channels in
// the same order as the stride-halving tree, so each bound is that tree's sum.
// Modes: per-row bounds of the active rows (one pass over a tile for up to
// kPcRows rows, else several), or the sparse-residual head score: per page the
// maximum of the bounds over every stacked row of the kv head (the four lanes
// of a page fold their rows with two shuffles; the running maximum of a page
// stays with one lane, which also folds it into the value stored by earlier
// blocks of staged rows).
// q rows are staged QR at a time as (q+ pair, q- pair) float4s; more rows
// repeat the page loop. Grid (tile ranges, Hkv, batch), one wave.
// ---------------------------------------------------------------------------
constexpr int kPcPages = 8;     // pages per warp tile
constexpr int kPcRows = 4;      // q rows per pass over a tile (kPcPages * kPcRows = 32)
constexpr int kPcStride = 34;   // float2 per transpose row: 272 bytes, conflict-free float4 reads
constexpr int kPcQRows = 64;      // q rows staged at a time (per-row bounds)
constexpr int kPcQRowsHead = 32;  // the same for the head score (two CTAs per SM)
constexpr int kPcThreads = 256;
constexpr int kPcRowsOnePass = 0;  // modes: per-row bounds, at most kPcRows rows
constexpr int kPcRowsMulti = 1;    //        per-row bounds, more rows
constexpr int kPcHeadMax = 2;      //        per-page maximum over every stacked row

__host__ __device__ constexpr int page_score_cols_smem(int RQ, int D, bool head_max) {
  return ((RQ < (head_max ? kPcQRowsHead : kPcQRows) ? (RQ + kPcRows - 1) / kPcRows * kPcRows
                                                     : (head_max ? kPcQRowsHead : kPcQRows)) *
          (D / 2) * 16) +
         (kPcThreads / 32) * 32 * kPcStride * 8;
}

template <int D, int kMode>
__global__ void __launch_bounds__(kPcThreads, 2)
    page_score_cols_kernel(const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ active,
                           const float* __restrict__ row_scores, int32_t* __restrict__ active_out,
                           int B, int Hq, int G, int n_act, const __nv_bfloat16* __restrict__ pmin,
                           const __nv_bfloat16* __restrict__ pmax, const KvView kv,
                           float* __restrict__ scores, uint32_t* __restrict__ bitmap, int words,
                           int* __restrict__ tickets, int tpc) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  static_assert(D % 64 == 0, "lanes hold D / 64 channel pairs");
  constexpr int NPL = D / 64;  // channel pairs per lane
  constexpr bool kOnePass = kMode == kPcRowsOnePass;
  constexpr bool kHeadMax = kMode == kPcHeadMax;
  constexpr int QR = kHeadMax ? kPcQRowsHead : kPcQRows;
  extern __shared__ __align__(16) float sm[];
  __shared__ int s_active[32];
  const int RQ = n_act * G;
  const int RQs = min((RQ + kPcRows - 1) / kPcRows * kPcRows, QR);  // staged rows
  float4* qpn = reinterpret_cast<float4*>(sm);                            // [RQs][D/2]
  float2* tr = reinterpret_cast<float2*>(qpn + RQs * (D / 2));            // [warps][32][stride]
  float* sc = reinterpret_cast<float*>(tr + (kPcThreads / 32) * 32 * kPcStride);  // [B] (pick)
  const int hk = blockIdx.y, b = blockIdx.z;
  if (blockIdx.x == 0) {
    for (int w = threadIdx.x; w < words; w += blockDim.x)
      bitmap[((long long)b * kv.Hkv + hk) * words + w] = 0u;
    if (tickets && threadIdx.x == 0) tickets[b * kv.Hkv + hk] = 0;
  }
  const int n_pages = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const int n_tiles = (n_pages + kPcPages - 1) / kPcPages;
  const int t0 = blockIdx.x * tpc, t1 = min(t0 + tpc, n_tiles);
  const bool pick = row_scores != nullptr;
  if (t0 >= t1 && !(pick && blockIdx.x == 0 && hk == 0)) return;
  const int* act = active ? active + b * n_act : nullptr;
  if (pick) {
    pick_active_rows(row_scores + (long long)b * B, B, n_act, sc, s_active);
    if (blockIdx.x == 0 && hk == 0)
      for (int r = threadIdx.x; r < n_act; r += blockDim.x) active_out[b * n_act + r] = s_active[r];
    if (t0 >= t1) return;
    act = s_active;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nw = kPcThreads / 32;
  float2* wtr = tr + warp * 32 * kPcStride;
  const __nv_bfloat16* mn0 = pmin + ((long long)b * kv.max_pages * kv.Hkv + hk) * D;
  const __nv_bfloat16* mx0 = pmax + ((long long)b * kv.max_pages * kv.Hkv + hk) * D;
  uint32_t dmn[kPcPages][NPL], dmx[kPcPages][NPL];
  // page pi of tile t: the clamped page is read for pages past the sequence
  // (their bounds are never stored), so every load is unconditional
  const int ps32 = kv.Hkv * (D / 2);  // 32-bit words from one page's row to the next
  const uint32_t* mn32 = reinterpret_cast<const uint32_t*>(mn0) + lane;
  const uint32_t* mx32 = reinterpret_cast<const uint32_t*>(mx0) + lane;
  auto load_page = [&](int pi, int t) {
    const int pc = min(t * kPcPages + pi, n_pages - 1);
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      dmn[pi][k] = __ldg(mn32 + pc * ps32 + 32 * k);
      dmx[pi][k] = __ldg(mx32 + pc * ps32 + 32 * k);
    }
  };
  float4 qv[kPcRows][NPL];
  auto load_q = [&](int r0) {
#pragma unroll
    for (int r = 0; r < kPcRows; ++r)
#pragma unroll
      for (int k = 0; k < NPL; ++k) qv[r][k] = qpn[(r0 + r) * (D / 2) + lane + 32 * k];
  };
  // one pass over a tile: the 32 bounds (kPcRows rows from staged row r0, the
  // tile's pages) up to the lane-local levels, into the transpose buffer. With
  // `reload`, each page's registers take page pi of tile tl as soon as they
  // are unpacked, so the next tile's loads overlap almost the whole pass.
  auto pass_bounds = [&](auto reload, int tl) {
#pragma unroll
    for (int pi = 0; pi < kPcPages; ++pi) {
      float2 n[NPL], x[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        n[k] = make_float2(__uint_as_float(dmn[pi][k] << 16),
                           __uint_as_float(dmn[pi][k] & 0xFFFF0000u));
        x[k] = make_float2(__uint_as_float(dmx[pi][k] << 16),
                           __uint_as_float(dmx[pi][k] & 0xFFFF0000u));
      }
      if constexpr (decltype(reload)::value) load_page(pi, tl);
#pragma unroll
      for (int r = 0; r < kPcRows; ++r) {
        float2 s[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k)
          s[k] = ffma2(make_float2(qv[r][k].z, qv[r][k].w), n[k],
                       fmul2(make_float2(qv[r][k].x, qv[r][k].y), x[k]));
#pragma unroll
        for (int st = NPL / 2; st >= 1; st >>= 1)  // channel strides D/2 .. 64
#pragma unroll
          for (int k = 0; k < st; ++k) s[k] = fadd2(s[k], s[k + st]);
        wtr[(r * kPcPages + pi) * kPcStride + lane] = s[0];
      }
    }
    __syncwarp();
  };
  // one pass: lane o's bound row (row o / kPcPages of rows 0..3), or NULL past RQ
  float* out_row = nullptr;
  if (kOnePass && lane / kPcPages < RQ) {
    const int rq = lane / kPcPages, a_i = rq / G, g = rq - (rq / G) * G;
    out_row = scores + (((long long)b * n_act + a_i) * Hq + hk * G + g) * kv.max_pages;
  }
  uint32_t hmax = 0u;  // head score: running maximum key of page (lane % kPcPages)
  // ... then lane o finishes bound o and stores it (head score: folds it)
  auto pass_finish = [&](int t, int r0, int row_base) {
    // float4 j of the row holds pairs 2j and 2j + 1 (channels 4j .. 4j + 3)
    const float4* row = reinterpret_cast<const float4*>(wtr + lane * kPcStride);
    float2 v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // channel strides 32 then 16: ((i + (i+16)) + ((i+8) + (i+24))) for pairs i = 2j, 2j + 1
      const float4 a = row[j], b8 = row[j + 4], c = row[j + 8], d = row[j + 12];
      v[2 * j] = fadd2(fadd2(make_float2(a.x, a.y), make_float2(c.x, c.y)),
                       fadd2(make_float2(b8.x, b8.y), make_float2(d.x, d.y)));
      v[2 * j + 1] = fadd2(fadd2(make_float2(a.z, a.w), make_float2(c.z, c.w)),
                           fadd2(make_float2(b8.z, b8.w), make_float2(d.z, d.w)));
    }
#pragma unroll
    for (int st = 4; st >= 1; st >>= 1)  // channel strides 8 .. 2
#pragma unroll
      for (int i = 0; i < st; ++i) v[i] = fadd2(v[i], v[i + st]);
    const float y = __fadd_rn(v[0].x, v[0].y);  // channel 0 + channel 1
    __syncwarp();  // the buffer is rewritten by the next pass
    const int p = t * kPcPages + (lane & (kPcPages - 1));
    if constexpr (kHeadMax) {
      const int rq = row_base + r0 + lane / kPcPages;
      uint32_t key = (p < n_pages && rq < RQ) ? order_key(y) : 0u;  // 0: below every key
      key = max(key, __shfl_xor_sync(0xffffffffu, key, kPcPages));
      key = max(key, __shfl_xor_sync(0xffffffffu, key, 2 * kPcPages));
      hmax = max(hmax, key);
    } else if (p < n_pages) {
      if constexpr (kOnePass) {
        if (out_row) out_row[p] = y;
      } else {
        const int rq = row_base + r0 + lane / kPcPages;
        if (rq < RQ) {
          const int a_i = rq / G, g = rq - (rq / G) * G;
          scores[(((long long)b * n_act + a_i) * Hq + hk * G + g) * kv.max_pages + p] = y;
        }
      }
    }
  };
  for (int row_base = 0; row_base < RQ; row_base += QR) {
    if (row_base > 0) __syncthreads();  // every warp is done with the previous rows
    for (int idx = threadIdx.x; idx < RQs * (D / 2); idx += blockDim.x) {
      const int rr = idx / (D / 2), c2 = idx - rr * (D / 2);
      const int rq = row_base + rr;
      float2 v = make_float2(0.f, 0.f);
      if (rq < RQ) {
        const int a_i = rq / G, g = rq - a_i * G;
        const int i = act ? act[a_i] : a_i;
        const uint32_t u = *reinterpret_cast<const uint32_t*>(
            q + (((long long)b * B + i) * Hq + hk * G + g) * D + 2 * c2);
        v = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
      }
      qpn[idx] = make_float4(v.x >= 0.f ? v.x : 0.f, v.y >= 0.f ? v.y : 0.f,
                             v.x < 0.f ? v.x : 0.f, v.y < 0.f ? v.y : 0.f);
    }
    __syncthreads();
    const int rows_here = min(RQ - row_base, QR);
    int t = t0 + warp;
    if (t < t1)
#pragma unroll
      for (int pi = 0; pi < kPcPages; ++pi) load_page(pi, t);
    if constexpr (kOnePass) load_q(0);
    for (; t < t1; t += nw) {
      // the last pass over a tile reloads the page registers with the next
      // tile (the warp's last tile reloads itself: the loads stay unconditional)
      const int tl = t + nw < t1 ? t + nw : t;
      if constexpr (kOnePass) {
        pass_bounds(std::true_type{}, tl);
        pass_finish(t, 0, row_base);
      } else {
        hmax = 0u;
        for (int r0 = 0; r0 < rows_here; r0 += kPcRows) {
          load_q(r0);
          if (r0 + kPcRows >= rows_here)
            pass_bounds(std::true_type{}, tl);
          else
            pass_bounds(std::false_type{}, tl);
          pass_finish(t, r0, row_base);
        }
        if constexpr (kHeadMax) {
          const int p = t * kPcPages + lane;
          if (lane < kPcPages && p < n_pages) {
            // the same lane holds this page in every block of staged rows
            float* dst = scores + ((long long)b * kv.Hkv + hk) * kv.max_pages + p;
            *dst = order_key_inv(row_base == 0 ? hmax : max(hmax, order_key(*dst)));
          }
        }
      }
    }
  }
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
constexpr int kTopkDigitBits = 12;  // radix digit width of the top-k select
constexpr int kTopkBinsPerThread = (1 << kTopkDigitBits) / kTopkThreads;
constexpr int kTopkLoads = 16;      // score loads in flight per thread

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
  __shared__ int hist[1 << kTopkDigitBits];
  __shared__ int warp_sums[33];
  __shared__ uint32_t s_prefix, s_kmin[kTopkThreads / 32], s_kmax[kTopkThreads / 32];
  __shared__ int s_need, s_neq, s_last;
  const int ah = blockIdx.x, b = blockIdx.y;
  const int h = ah % Hq;
  const int hk = h / G;
  const int tid = threadIdx.x;
  const int n = (kv_tokens(kv, b) + kv.page_size - 1) / kv.page_size;
  const int k = min(topk, n);
  uint32_t* sbm = keys + kv.max_pages;
  uint32_t* bm = bitmap + ((long long)b * kv.Hkv + hk) * words;
  const float* sc = scores + ((long long)b * n_act * Hq + ah) * kv.max_pages;
  const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (k <= 0) {
    for (int w = tid; w < words; w += blockDim.x) sbm[w] = 0u;
  } else if (k >= n) {  // every page of the sequence
    for (int w = tid; w < words; w += blockDim.x) {
      const int p0 = 32 * w;
      sbm[w] = p0 + 32 <= n ? 0xFFFFFFFFu : (p0 < n ? (1u << (n - p0)) - 1u : 0u);
    }
  } else {
    // The scores as order-preserving keys (a thread's loads all in flight at
    // once), with the smallest and largest key on the way.
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int p0 = tid; p0 < n; p0 += kTopkLoads * blockDim.x) {
      float v[kTopkLoads];
#pragma unroll
      for (int u = 0; u < kTopkLoads; ++u) {
        const int p = p0 + u * blockDim.x;
        v[u] = p < n ? __ldcg(sc + p) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kTopkLoads; ++u) {
        const int p = p0 + u * blockDim.x;
        if (p < n) {
          const uint32_t key = order_key(v[u]);
          keys[p] = key;
          lo = min(lo, key);
          hi = max(hi, key);
        }
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      s_kmin[warp] = lo;
      s_kmax[warp] = hi;
    }
    __syncthreads();
    lo = 0xFFFFFFFFu;
    hi = 0u;
    for (int w = 0; w < nw; ++w) {
      lo = min(lo, s_kmin[w]);
      hi = max(hi, s_kmax[w]);
    }
    // Radix select of the k-th largest key T. The bits every key shares (the
    // common prefix of the smallest and largest key) are fixed at once; the
    // rest are resolved kTopkDigitBits at a time, most significant first, each
    // pass counting only the keys that match the bits fixed so far.
    int free_bits = (lo ^ hi) ? 32 - __clz(lo ^ hi) : 0;  // bits below the common prefix
    uint32_t mask = free_bits == 32 ? 0u : ~((1u << free_bits) - 1u);
    uint32_t prefix = hi & mask;
    int need = k;   // keys equal to the prefix still to take
    int n_eq = n;   // keys equal to the prefix
    while (free_bits > 0) {
      const int w = free_bits < kTopkDigitBits ? free_bits : kTopkDigitBits;
      const int shift = free_bits - w;
      const int nb = 1 << w;
      for (int d = tid; d < nb; d += blockDim.x) hist[d] = 0;
      __syncthreads();
      for (int p = tid; p < n; p += blockDim.x) {
        const uint32_t key = keys[p];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
      }
      __syncthreads();
      // digits in descending order: thread t owns the kTopkBinsPerThread
      // digits below nb - 1 - t * kTopkBinsPerThread
      int cnt[kTopkBinsPerThread], tot = 0;
#pragma unroll
      for (int j = 0; j < kTopkBinsPerThread; ++j) {
        const int d = nb - 1 - tid * kTopkBinsPerThread - j;
        cnt[j] = d >= 0 ? hist[d] : 0;
        tot += cnt[j];
      }
      int total;
      const int before = block_exclusive_scan(tot, warp_sums, total);
      if (before < need && before + tot >= need) {  // exactly one thread
        int cum = before;
#pragma unroll
        for (int j = 0; j < kTopkBinsPerThread; ++j) {
          if (cum + cnt[j] >= need) {
            s_prefix = prefix | ((uint32_t)(nb - 1 - tid * kTopkBinsPerThread - j) << shift);
            s_need = need - cum;
            s_neq = cnt[j];
            break;
          }
          cum += cnt[j];
        }
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      n_eq = s_neq;
      mask |= (uint32_t)(nb - 1) << shift;
      free_bits = shift;
    }
    const uint32_t T = prefix;  // the k-th largest key; `need` of the n_eq keys equal to it are taken
    // Selection words, one per warp step (bit i of word w: page 32 w + i): every
    // key above T, and the keys equal to T -- all of them, or where more equal
    // T than are taken, the lowest pages.
    if (n_eq == need) {
      for (int w = warp; w < words; w += nw) {
        const int p = 32 * w + lane;
        const unsigned bits = __ballot_sync(0xffffffffu, p < n && keys[p] >= T);
        if (lane == 0) sbm[w] = bits;
      }
    } else {
      for (int w = warp; w < words; w += nw) {  // equal keys per word
        const int p = 32 * w + lane;
        const unsigned eq = __ballot_sync(0xffffffffu, p < n && keys[p] == T);
        if (lane == 0) hist[w] = __popc(eq);
      }
      __syncthreads();
      const int per = (words + blockDim.x - 1) / blockDim.x;  // words per thread, in order
      const int w0 = tid * per, w1 = min(words, w0 + per);
      int c = 0;
      for (int w = w0; w < w1; ++w) c += hist[w];
      int total;
      int before = block_exclusive_scan(c, warp_sums, total);
      for (int w = w0; w < w1; ++w) {  // equal keys in the words before w
        const int cw = hist[w];
        hist[w] = before;
        before += cw;
      }
      __syncthreads();
      for (int w = warp; w < words; w += nw) {
        const int p = 32 * w + lane;
        const uint32_t key = p < n ? keys[p] : 0u;
        const unsigned gt = __ballot_sync(0xffffffffu, p < n && key > T);
        unsigned eq = __ballot_sync(0xffffffffu, p < n && key == T);
        if (lane == 0) {
          unsigned take = 0u;
          for (int left = need - hist[w]; left > 0 && eq; --left) {
            const unsigned low = eq & (0u - eq);  // lowest equal page of the word
            take |= low;
            eq ^= low;
          }
          sbm[w] = gt | take;
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
// max(q_c kmin_c, q_c kmax_c). For float32 summaries (bf16: the head-score mode
// of page_score_cols_kernel) the per-(row, head) bound is formed exactly as in
// page_score_kernel (single-rounded products, stride-halving tree); the maximum
// is order-free, taken on order-preserving keys with shared-memory atomics.
// scores: [batch, Hkv, max_pages]. Block (0, hk, b) clears the (b, hk) bitmap.
// Rows are taken kHsRows at a time (q staged per group, every page chunk
// streamed again per group, from L2 where it fits): the maximum is order-free,
// and later groups fold theirs into the scores the earlier groups wrote.
// ---------------------------------------------------------------------------
constexpr int kHsRows = 64;


template <typename T, int D>
__global__ void __launch_bounds__(256, 2)
    head_page_score_kernel(const T* __restrict__ q, int B, int Hq, int G,
                           const T* __restrict__ pmin, const T* __restrict__ pmax,
                           const KvView kv, float* __restrict__ scores,
                           uint32_t* __restrict__ bitmap, int words, int* __restrict__ tickets,
                           int cpc) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  static_assert(sizeof(T) == 4, "float32 summaries (bf16: page_score_cols_kernel)");
  constexpr int PS = ps_stride<T, D>();
  extern __shared__ __align__(16) float sm[];
  __shared__ uint32_t best[kPsPages];
  const int RQ_all = B * G;
  const int RQmax = RQ_all < kHsRows ? RQ_all : kHsRows;
  float* qs = sm;                                  // [RQmax][D], row r = i * G + g
  T* sbuf = reinterpret_cast<T*>(qs + RQmax * D);  // stages of [64][PS]
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
  for (int row0 = 0; row0 < RQ_all; row0 += kHsRows) {
  const int RQ = RQ_all - row0 < kHsRows ? RQ_all - row0 : kHsRows;
  ring.prologue();
  stage_q_rows<T, D>(q, nullptr, b, B, Hq, G, hk, B, RQ, qs, row0);
  for (int ch = c0; ch < c1; ++ch) {
    for (int pg = threadIdx.x; pg < kPsPages; pg += blockDim.x) best[pg] = 0u;  // below every key
    ring.advance(ch);
    const T* smn = ring.mn(ch);
    const T* smx = ring.mx(ch);
    __syncthreads();  // chunk ch, the q rows and the cleared maxima visible to every thread
    for (int task = threadIdx.x; task < kPsPages * RQ; task += blockDim.x) {
      const int pg = task % kPsPages, rq = task / kPsPages;
      const int p = ch * kPsPages + pg;
      if (p >= n_pages) continue;
      const float yb = page_bound<T, D>(qs + rq * D, smn + pg * PS, smx + pg * PS);
      atomicMax(&best[pg], order_key(yb));
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
