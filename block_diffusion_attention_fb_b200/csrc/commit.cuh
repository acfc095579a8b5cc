// Block commit: a finished block's keys and values join the block-external
// cache, and the per-page key summaries of the LoSA selector follow.
//
// Block diffusion generates causally between blocks (FlashBlock abstract and
// technical summary §2): once block k is final its tokens are part of J_out
// for block k+1. Sequence b with n_b tokens receives block row j at position
// n_b + j, in the cache's own addressing (page table or contiguous rows). The
// summaries (LoSA §2 step 3: per page, kv head and channel, min and max of the
// page's keys) change only on pages that receive tokens: a page that already
// held tokens combines its old summary with the new keys, a fresh page takes
// the new keys alone. min and max are exact, so the incremental result equals
// a summary recomputed from scratch bit for bit.
//
// One CTA per (touched page of a sequence, kv head, sequence) copies the
// page's new K and V rows with 16-byte loads, all issued before any store,
// then folds the new keys into the summary per channel. The new lengths come
// from the host (the caller tracks them to map pages), so nothing here reads
// the device lengths that it updates.
#pragma once

#include "common.cuh"

namespace fb {

constexpr int kMaxCommitBatch = 256;

struct CommitArgs {
  const void* k_in;  // [batch, B, Hkv, D] block rows
  const void* v_in;
  void* k;  // [n_slots, Hkv, D] cache pool
  void* v;
  const int32_t* page_table;  // [batch, max_pages] or NULL (contiguous)
  int32_t* seq_len;           // [batch] device lengths (written: n_b + B)
  void* pmin;                 // [batch, max_pages, Hkv, D] or NULL (no summaries kept)
  void* pmax;
  long long n_slots;
  int batch, B, Hkv, page_size, max_pages, max_seq_len;
  int n_old[kMaxCommitBatch];  // lengths before the call
};

// A page-table entry outside the pool sets kErrBadPage (common.cuh) and the
// page is left unwritten; fb_device_status reports it.

template <typename T>
__device__ __forceinline__ float commit_f32(T x);
template <>
__device__ __forceinline__ float commit_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float commit_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T commit_from_f32(float x);
template <>
__device__ __forceinline__ float commit_from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 commit_from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);  // exact: x is a bf16 value
}

// One CTA of 256 threads per (touched page, kv head, sequence). Thread
// (token slot u, 16-byte chunk v) moves one chunk of K and one of V; every
// load of the page is issued before any store (one memory round trip). The
// summary is then folded per channel from the K rows staged in shared memory.
constexpr int kCommitThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kCommitThreads)
    block_commit_kernel(const __grid_constant__ CommitArgs a) {
  constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  constexpr int CH = D / VE;               // chunks per row
  extern __shared__ uint4 srows[];         // [page tokens][CH] new K rows
  const int pi = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int n = a.n_old[b], P = a.page_size;
  const int p = n / P + pi;  // logical page
  const int t0 = max(n, p * P), t1 = min(n + a.B, (p + 1) * P);
  if (pi == 0 && hk == 0 && tid == 0 && a.seq_len) a.seq_len[b] = n + a.B;
  if (t0 >= t1) return;
  long long page_slot = (long long)b * a.max_seq_len + (long long)p * P;
  if (a.page_table) {
    const int pg = a.page_table[(long long)b * a.max_pages + p];
    if (pg < 0 || ((long long)pg + 1) * P > a.n_slots) {  // unmapped or outside the pool
      if (tid == 0) atomicOr(&g_fb_error_word, kErrBadPage);
      return;
    }
    page_slot = (long long)pg * P;
  }
  const uint4* __restrict__ kin = static_cast<const uint4*>(a.k_in);
  const uint4* __restrict__ vin = static_cast<const uint4*>(a.v_in);
  uint4* __restrict__ kc = static_cast<uint4*>(a.k);
  uint4* __restrict__ vc = static_cast<uint4*>(a.v);
  const int nt = t1 - t0, total = nt * CH;
  // at most 4 chunks of K and V per thread in flight at once
  for (int base = 0; base < total; base += 4 * kCommitThreads) {
    uint4 kx[4], vx[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = base + r * kCommitThreads + tid;
      if (idx < total) {
        const int u = idx / CH, v = idx - u * CH;
        const long long src = (((long long)b * a.B + (t0 + u - n)) * a.Hkv + hk) * CH + v;
        kx[r] = kin[src];
        vx[r] = vin[src];
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = base + r * kCommitThreads + tid;
      if (idx < total) {
        const int u = idx / CH, v = idx - u * CH;
        const long long dst = ((page_slot + (t0 + u - p * P)) * a.Hkv + hk) * CH + v;
        kc[dst] = kx[r];
        vc[dst] = vx[r];
        srows[u * CH + v] = kx[r];
      }
    }
  }
  if (!a.pmin) return;
  __syncthreads();
  const T* sk = reinterpret_cast<const T*>(srows);
  T* smin = static_cast<T*>(a.pmin);
  T* smax = static_cast<T*>(a.pmax);
  for (int c = tid; c < D; c += kCommitThreads) {
    float mn = INFINITY, mx = -INFINITY;
    for (int u = 0; u < nt; ++u) {
      const float f = commit_f32<T>(sk[u * D + c]);
      mn = fminf(mn, f);
      mx = fmaxf(mx, f);
    }
    const long long o = (((long long)b * a.max_pages + p) * a.Hkv + hk) * D + c;
    if (n > p * P) {  // the page already held tokens: fold in its summary
      mn = fminf(mn, commit_f32<T>(smin[o]));
      mx = fmaxf(mx, commit_f32<T>(smax[o]));
    }
    smin[o] = commit_from_f32<T>(mn);
    smax[o] = commit_from_f32<T>(mx);
  }
}

}  // namespace fb
