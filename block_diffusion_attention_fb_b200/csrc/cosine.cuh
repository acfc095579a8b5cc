// Per-head similarity for FlashBlock's per-head reuse in video diffusion
// (technical summary, §2 "Adaptive reuse strategies": only heads whose
// similarity is above gamma reuse the cache).
//
// c_h = cos(A_out,h^s, A_out,h^{s-1}) over the head's flattened B x d tile, in
// float64: products of float32 values are exact in float64; the three sums
// (dot, |a|^2, |b|^2) follow the stride-halving tree over n = i * d + c padded
// with zeros to a power of two P; c = dot / sqrt(|a|^2 |b|^2) (0 if either
// tile is zero). Stage 1: T1 = min(P, 16384) threads per head, each owning
// n = t + j * T1 and reducing over j in tree order; stage 2: one CTA per head
// finishes the tree over t and updates the head's compute mask (sticky reuse
// once c >= gamma).
#pragma once

#include "common.cuh"

namespace fb {

constexpr int kCosT1Max = 16384;
constexpr int kCosEMax = 16;  // P <= 16384 * 16 = 262144 elements per head

__global__ void __launch_bounds__(256)
    head_cos_stage1(const float* __restrict__ cur, const float* __restrict__ prev,
                    const uint8_t* __restrict__ mask, int B, int Hq, int D, int N, int T1, int E,
                    double* __restrict__ part) {
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh - (bh / Hq) * Hq;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T1) return;
  if (!mask[bh]) return;
  double dd[kCosEMax], aa[kCosEMax], bb[kCosEMax];
#pragma unroll
  for (int j = 0; j < kCosEMax; ++j) {
    dd[j] = aa[j] = bb[j] = 0.0;
    if (j < E) {
      const int n = t + j * T1;
      if (n < N) {
        const int i = n / D, c = n - (n / D) * D;
        const long long off = (((long long)b * B + i) * Hq + h) * D + c;
        const double x = cur[off], y = prev[off];
        dd[j] = __dmul_rn(x, y);
        aa[j] = __dmul_rn(x, x);
        bb[j] = __dmul_rn(y, y);
      }
    }
  }
#pragma unroll
  for (int s = kCosEMax / 2; s >= 1; s >>= 1) {
    if (s < E) {
#pragma unroll
      for (int j = 0; j < s; ++j) {
        dd[j] = __dadd_rn(dd[j], dd[j + s]);
        aa[j] = __dadd_rn(aa[j], aa[j + s]);
        bb[j] = __dadd_rn(bb[j], bb[j + s]);
      }
    }
  }
  double* p = part + (long long)bh * 3 * T1;
  p[t] = dd[0];
  p[T1 + t] = aa[0];
  p[2 * T1 + t] = bb[0];
}

__global__ void __launch_bounds__(1024)
    head_cos_stage2(const double* __restrict__ part, int T1, double gamma,
                    uint8_t* __restrict__ mask, double* __restrict__ head_cos) {
  __shared__ double sd[1024], sa[1024], sb[1024];
  const int bh = blockIdx.x, tid = threadIdx.x;
  if (!mask[bh]) {  // a head that did not compute this step has no new cosine
    if (tid == 0) head_cos[bh] = __longlong_as_double(0x7ff8000000000000LL);
    return;
  }
  const int T2 = T1 < 1024 ? T1 : 1024;
  const int E2 = T1 / T2;
  const double* p = part + (long long)bh * 3 * T1;
  if (tid < T2) {
    double d[kCosEMax], a[kCosEMax], b[kCosEMax];
#pragma unroll
    for (int j = 0; j < kCosEMax; ++j) {
      d[j] = a[j] = b[j] = 0.0;
      if (j < E2) {
        d[j] = p[tid + j * T2];
        a[j] = p[T1 + tid + j * T2];
        b[j] = p[2 * T1 + tid + j * T2];
      }
    }
#pragma unroll
    for (int s = kCosEMax / 2; s >= 1; s >>= 1) {
      if (s < E2) {
#pragma unroll
        for (int j = 0; j < s; ++j) {
          d[j] = __dadd_rn(d[j], d[j + s]);
          a[j] = __dadd_rn(a[j], a[j + s]);
          b[j] = __dadd_rn(b[j], b[j + s]);
        }
      }
    }
    sd[tid] = d[0];
    sa[tid] = a[0];
    sb[tid] = b[0];
  }
  __syncthreads();
  for (int s = T2 >> 1; s >= 1; s >>= 1) {
    if (tid < s) {
      sd[tid] = __dadd_rn(sd[tid], sd[tid + s]);
      sa[tid] = __dadd_rn(sa[tid], sa[tid + s]);
      sb[tid] = __dadd_rn(sb[tid], sb[tid + s]);
    }
    __syncthreads();
  }
  if (tid == 0) {
    const double den = __dmul_rn(sa[0], sb[0]);
    const double c = den == 0.0 ? 0.0 : __ddiv_rn(sd[0], __dsqrt_rn(den));
    head_cos[bh] = c;
    if (c >= gamma) mask[bh] = 0;
  }
}

}  // namespace fb
