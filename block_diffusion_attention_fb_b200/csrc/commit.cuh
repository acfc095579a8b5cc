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
// One CTA per (touched page of a sequence, kv head, sequence), one thread per
// channel: it copies the page's new K and V rows (coalesced across channels)
// and folds the new keys into the summary in registers. The new lengths come
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

// Error-word bit set when a page-table entry points outside the pool (the
// page is then left unwritten); fb_device_status reports it.
constexpr int kErrBadPage = 2;

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

template <typename T, int D>
__global__ void __launch_bounds__(D) block_commit_kernel(const __grid_constant__ CommitArgs a) {
  const int pi = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
  const int n = a.n_old[b], P = a.page_size;
  const int p = n / P + pi;  // logical page
  const int t0 = max(n, p * P), t1 = min(n + a.B, (p + 1) * P);
  if (pi == 0 && hk == 0 && c == 0 && a.seq_len) a.seq_len[b] = n + a.B;
  if (t0 >= t1) return;
  long long page_slot = (long long)b * a.max_seq_len + (long long)p * P;
  if (a.page_table) {
    const int pg = a.page_table[(long long)b * a.max_pages + p];
    if (pg < 0 || ((long long)pg + 1) * P > a.n_slots) {  // unmapped or outside the pool
      if (c == 0) atomicOr(&g_fb_error_word, kErrBadPage);
      return;
    }
    page_slot = (long long)pg * P;
  }
  const T* kin = static_cast<const T*>(a.k_in);
  const T* vin = static_cast<const T*>(a.v_in);
  T* kc = static_cast<T*>(a.k);
  T* vc = static_cast<T*>(a.v);
  float mn = INFINITY, mx = -INFINITY;
  for (int t = t0; t < t1; ++t) {
    const long long src = (((long long)b * a.B + (t - n)) * a.Hkv + hk) * D + c;
    const long long dst = ((page_slot + (t - p * P)) * a.Hkv + hk) * D + c;
    const T kx = kin[src];
    kc[dst] = kx;
    vc[dst] = vin[src];
    const float f = commit_f32<T>(kx);
    mn = fminf(mn, f);
    mx = fmaxf(mx, f);
  }
  if (a.pmin) {
    T* smin = static_cast<T*>(a.pmin);
    T* smax = static_cast<T*>(a.pmax);
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
