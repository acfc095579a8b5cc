// Block-internal partial (A_in, L_in) for short blocks, optionally fused with
// the FlashBlock log-space merge against the cached block-external partial
// (FlashBlock technical summary, §2 "Core mechanism": the in-block part is
// recomputed every denoising step, then combined with the cached
// (A_out, L_out) by m = max(L_out, L_in), w_x = e^{L_x - m},
// A_full = (w_out A_out + w_in A_in) / (w_out + w_in)).
//
// The key set is the block's own B <= 64 tokens, bidirectional (every block
// row sees every block key). The work is tiny (dLLM block of 32: 0.5 MFLOP per
// head) and the call sits on every denoising step, so the kernel is built for
// latency, not throughput:
//   * one CTA per (sequence, kv head, tile of 16 x warps stacked query rows);
//   * every input it needs -- its Q rows, the kv head's K and V rows and the
//     merge partner rows -- is requested at once with cp.async (16-byte
//     chunks, zero-filled past the block), so the CTA pays one memory round
//     trip before computing;
//   * one pass, no pipeline: the whole key set fits in one tile, so the
//     softmax is exact (row maximum over all keys, then exponentials);
//   * QK^T and PV on bf16 tensor cores (mma.sync m16n8k16, fp32 accumulate)
//     with ldmatrix fragment loads from padded shared rows (no bank
//     conflicts); P stays in registers between the two products.
// GQA q heads sharing a kv head are stacked as rows r = i * G + g.
#pragma once

#include "common.cuh"

namespace fb {

struct BlockArgs {
  const __nv_bfloat16* q;  // [batch, B, Hq, D], or [total, Hq, D] packed (cu)
  const __nv_bfloat16* k;  // [batch, B, Hkv, D], or [total, Hkv, D] packed
  const __nv_bfloat16* v;
  const int32_t* cu;       // packed rows: sequence b owns rows cu[b] .. cu[b+1]-1, or NULL
  int total;               // rows of the packed buffers
  const float* mrg_a;  // [batch, B, Hq, D] cached block-external partial, or NULL (no merge)
  const float* mrg_l;  // [batch, B, Hq]
  float* a_out;        // [batch, B, Hq, D]: A_in, or A_full with the merge
  float* l_out;        // [batch, B, Hq]: natural log
  int batch, B, Hq, Hkv, G, R;  // R = B * G rows per (sequence, kv head); packed: B = most rows
  float scale_log2;
};

// First row and row count of sequence b (packed or batched layout).
template <typename Args>
__device__ __forceinline__ int block_rows(const Args& a, int b, long long& base) {
  if (!a.cu) {
    base = (long long)b * a.B;
    return a.B;
  }
  return packed_range(a.cu, b, a.total, a.B, base);
}

template <int D>
struct BlockSmem {
  static constexpr int kRowB = D * 2 + 16;  // bf16 row: +16 B so ldmatrix rows hit distinct banks
  static constexpr int kRowM = D * 4 + 32;  // fp32 merge row: float2 reads of a half warp are conflict-free
  static int bytes(int warps, int key_tiles, bool merge) {
    const int rows = warps * 16;
    return rows * kRowB + 2 * key_tiles * 16 * kRowB + (merge ? rows * kRowM : 0);
  }
};

// KT: key tiles of 16 (the block's B keys padded to 16 * KT <= 64).
template <int D, int KT>
__global__ void __launch_bounds__(128) block_attn_kernel(const __grid_constant__ BlockArgs a) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  using S = BlockSmem<D>;
  constexpr int NT = 2 * KT;  // n8 tiles of keys
  constexpr int KD = D / 16;  // k16 steps over the head dim
  constexpr int NK = 16 * KT;
  extern __shared__ __align__(16) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthr = blockDim.x, RT = (nthr >> 5) * 16;
  const int rt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int row0 = rt * RT;
  const bool merge = a.mrg_a != nullptr;
  long long base;
  const int Bb = block_rows(a, b, base);  // block rows (= keys) of this sequence
  const int Rb = Bb * a.G;

  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + RT * S::kRowB;
  const uint32_t sV = sK + NK * S::kRowB;
  const uint32_t sM = sV + NK * S::kRowB;
  const float* mrow_base = reinterpret_cast<const float*>(smem + (sM - sQ));

  // ---- one round of loads: Q rows, K and V of the block, then merge rows ----
  constexpr int C8 = D / 8;  // 16-byte chunks of a bf16 row
  for (int idx = tid; idx < RT * C8; idx += nthr) {
    const int rl = idx / C8, c = idx - rl * C8;
    const int r = row0 + rl;
    const __nv_bfloat16* src = a.q;
    uint32_t nb = 0;
    if (r < Rb) {
      const int i = r / a.G, h = hk * a.G + (r - i * a.G);
      src = a.q + ((base + i) * a.Hq + h) * D + c * 8;
      nb = 16;
    }
    cp_async16(sQ + rl * S::kRowB + c * 16, src, nb);
  }
  for (int idx = tid; idx < NK * C8; idx += nthr) {
    const int j = idx / C8, c = idx - j * C8;
    const long long off = ((base + j) * a.Hkv + hk) * D + c * 8;
    const bool ok = j < Bb;  // keys past the block are zero-filled (and masked below)
    cp_async16(sK + j * S::kRowB + c * 16, ok ? a.k + off : a.k, ok ? 16u : 0u);
    cp_async16(sV + j * S::kRowB + c * 16, ok ? a.v + off : a.v, ok ? 16u : 0u);
  }
  cp_async_commit();
  if (merge) {
    // each warp loads the merge rows of its own 16 rows, so a __syncwarp
    // after its wait is enough before reading them
    constexpr int C4 = D / 4;  // 16-byte chunks of an fp32 row
    for (int idx = lane; idx < 16 * C4; idx += 32) {
      const int rl = warp * 16 + idx / C4, c = idx % C4;
      const int r = row0 + rl;
      const float* src = a.mrg_a;
      uint32_t nb = 0;
      if (r < Rb) {
        const int i = r / a.G, h = hk * a.G + (r - i * a.G);
        src = a.mrg_a + ((base + i) * a.Hq + h) * D + c * 4;
        nb = 16;
      }
      cp_async16(sM + rl * S::kRowM + c * 16, src, nb);
    }
  }
  cp_async_commit();

  // rows of this thread: g8 and g8 + 8 of the warp's 16
  const int g8 = lane >> 2, t4 = lane & 3;
  const int wrow0 = row0 + warp * 16;
  long long grow[2] = {-1, -1};  // [batch, B, Hq] row index of the output
  float Lo[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int r = wrow0 + g8 + hr * 8;
    if (r < Rb) {
      const int i = r / a.G, h = hk * a.G + (r - i * a.G);
      grow[hr] = (base + i) * a.Hq + h;
      if (merge) Lo[hr] = __ldg(a.mrg_l + grow[hr]);
    }
  }

  cp_async_wait<1>();  // Q, K, V of this thread landed
  __syncthreads();     // ... and every other thread's
  if (wrow0 >= Rb) {
    cp_async_wait<0>();  // no copy of this thread outlives it
    return;
  }

  // ---------------------------- S = Q K^T ----------------------------------
  const int mi = lane >> 3, r8 = lane & 7;
  float s[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KD; ++kk) {
    uint32_t qa[4];
    ldsm_x4(sQ + (warp * 16 + (mi & 1) * 8 + r8) * S::kRowB + (2 * kk + (mi >> 1)) * 16, qa[0],
            qa[1], qa[2], qa[3]);
#pragma unroll
    for (int np = 0; np < KT; ++np) {
      const int key = np * 16 + (mi >> 1) * 8 + r8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + key * S::kRowB + (2 * kk + (mi & 1)) * 16, b0, b1, b2, b3);
      mma_bf16(s[2 * np], qa, b0, b1);
      mma_bf16(s[2 * np + 1], qa, b2, b3);
    }
  }
  // ------------------------ exact softmax over the block ------------------------
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = n * 8 + 2 * t4 + (e & 1);
      const float x = key < Bb ? s[n][e] * a.scale_log2 : -INFINITY;
      s[n][e] = x;
      mx[e >> 1] = fmaxf(mx[e >> 1], x);
    }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
  }
  const float bse[2] = {mx[0] == -INFINITY ? 0.f : mx[0], mx[1] == -INFINITY ? 0.f : mx[1]};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s[n][e] = fast_exp2(s[n][e] - bse[e >> 1]);
      rs[e >> 1] += s[n][e];
    }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 1);
    rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 2);
  }
  // ------------------------------ O = P V ---------------------------------
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll
  for (int kst = 0; kst < KT; ++kst) {
    const uint32_t pa[4] = {pack_bf16(s[2 * kst][0], s[2 * kst][1]),
                            pack_bf16(s[2 * kst][2], s[2 * kst][3]),
                            pack_bf16(s[2 * kst + 1][0], s[2 * kst + 1][1]),
                            pack_bf16(s[2 * kst + 1][2], s[2 * kst + 1][3])};
#pragma unroll
    for (int dp = 0; dp < D / 16; ++dp) {
      const int key = kst * 16 + (mi & 1) * 8 + r8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sV + key * S::kRowB + (2 * dp + (mi >> 1)) * 16, b0, b1, b2, b3);
      mma_bf16(o[2 * dp], pa, b0, b1);
      mma_bf16(o[2 * dp + 1], pa, b2, b3);
    }
  }

  // ------------------- normalise, merge, write A and L ---------------------
  cp_async_wait<0>();  // this thread's merge rows landed
  __syncwarp();        // ... and those of the warp (a warp reads only its own 16 rows)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    if (grow[hr] < 0) continue;
    const float Ln = rs[hr] > 0.f ? (bse[hr] + log2f(rs[hr])) * kLn2 : -INFINITY;
    float wn = rs[hr] > 0.f ? 1.f / rs[hr] : 0.f, wo = 0.f, L = Ln;
    if (merge) {
      const float m = fmaxf(Lo[hr], Ln);
      if (m == -INFINITY) {
        wn = 0.f;
        L = -INFINITY;
      } else {
        const float eo = expf(Lo[hr] - m), en = expf(Ln - m);
        const float inv = 1.f / (eo + en);
        wn *= en * inv;  // the in-block rows are still unnormalised: fold 1 / l in
        wo = eo * inv;
        L = m + logf(eo + en);
      }
    }
    const float* mrow = mrow_base + (warp * 16 + g8 + hr * 8) * (S::kRowM / 4);
    float* dst = a.a_out + grow[hr] * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int col = n * 8 + 2 * t4;
      float x0 = wn > 0.f ? wn * o[n][2 * hr] : 0.f;
      float x1 = wn > 0.f ? wn * o[n][2 * hr + 1] : 0.f;
      if (wo > 0.f) {  // a side with weight 0 is not read (it may hold stale bits)
        const float2 u = *reinterpret_cast<const float2*>(mrow + col);
        x0 += wo * u.x;
        x1 += wo * u.y;
      }
      *reinterpret_cast<float2*>(dst + col) = make_float2(x0, x1);
    }
    if (t4 == 0) a.l_out[grow[hr]] = L;
  }
}

// ---------------------------------------------------------------------------
// fp32 inputs (the same short-block role, float32 arithmetic throughout, no
// tensor cores): one CTA per (sequence, kv head). K (stored transposed, so the
// lanes of a warp read consecutive keys), V and the stacked Q rows are staged
// with cp.async in one round trip; warp w takes rows w, w + 8, ...: lane j
// forms s_j and s_{j+32} by fp32 FMA over the channels, the row maximum and sum
// come from warp shuffles, and lane j accumulates output channels j, j + 32, ...
// The FlashBlock merge with the cached partial is fused as in the bf16 kernel.
// ---------------------------------------------------------------------------
struct BlockArgsF32 {
  const float* q;  // [batch, B, Hq, D], or packed as in BlockArgs
  const float* k;  // [batch, B, Hkv, D]
  const float* v;
  const int32_t* cu;
  int total;
  const float* mrg_a;
  const float* mrg_l;
  float* a_out;
  float* l_out;
  int batch, B, Hq, Hkv, G, R;
  float scale;
};

// shared memory of block_attn_f32_kernel for R stacked rows
constexpr int block_f32_smem(int D, int R) { return 4 * D * (64 + R + 65); }

template <int D>
__global__ void __launch_bounds__(256) block_attn_f32_kernel(const __grid_constant__ BlockArgsF32 a) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  constexpr int NK = 64;       // keys staged (B <= 64)
  constexpr int KP = NK + 1;   // padded stride of the transposed keys: no bank conflicts
  extern __shared__ __align__(16) float fsm[];
  float* vs = fsm;             // [NK][D]
  float* qs = vs + NK * D;     // [R][D]
  float* kT = qs + a.R * D;    // [D][KP]
  const int hk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  long long base;
  const int Bb = block_rows(a, b, base);  // block rows (= keys) of this sequence
  const int Rb = Bb * a.G;                // a.R (the most rows) sizes the shared layout
  // V and Q rows by cp.async (16-byte chunks), K through registers into the
  // transposed layout; keys past the block are zero
  constexpr int C4 = D / 4;
  for (int idx = tid; idx < NK * C4; idx += blockDim.x) {
    const int j = idx / C4, c = idx - j * C4;
    const bool ok = j < Bb;
    const long long off = ((base + (ok ? j : 0)) * a.Hkv + hk) * D + c * 4;
    cp_async16(smem_u32(vs + j * D + c * 4), a.v + off, ok ? 16u : 0u);
  }
  for (int idx = tid; idx < Rb * C4; idx += blockDim.x) {
    const int r = idx / C4, c = idx - r * C4;
    const int i = r / a.G, h = hk * a.G + (r - i * a.G);
    cp_async16(smem_u32(qs + r * D + c * 4), a.q + ((base + i) * a.Hq + h) * D + c * 4,
               16u);
  }
  cp_async_commit();
  for (int idx = tid; idx < NK * D; idx += blockDim.x) {
    const int j = idx / D, c = idx - j * D;
    kT[c * KP + j] = j < Bb ? a.k[((base + j) * a.Hkv + hk) * D + c] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();
  constexpr int NV = D / 32;
  for (int r = warp; r < Rb; r += nw) {
    const float* qr = qs + r * D;
    float s0 = 0.f, s1 = 0.f;  // keys lane and lane + 32
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float qc = qr[c];
      s0 = fmaf(qc, kT[c * KP + lane], s0);
      s1 = fmaf(qc, kT[c * KP + lane + 32], s1);
    }
    s0 = lane < Bb ? s0 * a.scale : -INFINITY;
    s1 = lane + 32 < Bb ? s1 * a.scale : -INFINITY;
    float m = fmaxf(s0, s1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float p0 = expf(s0 - m), p1 = expf(s1 - m);  // the block has >= 1 key: m finite
    float l = p0 + p1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    float o[NV];
#pragma unroll
    for (int t = 0; t < NV; ++t) o[t] = 0.f;
    for (int j = 0; j < Bb; ++j) {
      const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
      for (int t = 0; t < NV; ++t) o[t] = fmaf(pj, vs[j * D + lane + 32 * t], o[t]);
    }
    const int i = r / a.G, h = hk * a.G + (r - i * a.G);
    const long long row = (base + i) * a.Hq + h;
    const float Ln = m + logf(l);
    float wn = 1.f / l, wo = 0.f, L = Ln;
    if (a.mrg_a) {
      const float Lo = a.mrg_l[row];
      const float mm = fmaxf(Lo, Ln);
      const float eo = expf(Lo - mm), en = expf(Ln - mm);  // Ln finite, so mm is
      const float inv = 1.f / (eo + en);
      wn *= en * inv;
      wo = eo * inv;
      L = mm + logf(eo + en);
    }
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      const int col = lane + 32 * t;
      float x = wn * o[t];
      if (wo > 0.f) x += wo * a.mrg_a[row * D + col];  // a side with weight 0 is not read
      a.a_out[row * D + col] = x;
    }
    if (lane == 0) a.l_out[row] = L;
  }
}

}  // namespace fb
