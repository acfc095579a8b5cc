// Attention partial on the 5th-generation tensor cores (tcgen05), head_dim 128.
//
// Same work split and outputs as attn_bf16_kernel (one CTA per split, kv head,
// sequence and row tile; GQA q heads stacked into the rows), but the two
// contractions run as asynchronous tcgen05.mma with fp32 accumulators in TMEM:
//   S_j = Q K_j^T   (M = 128 rows, N = 64 keys, K = 128 channels) -> TMEM
//   O  += P_j V_j   (M = 128 rows, N = 128 channels, K = 64 keys)  -> TMEM
// Warp roles (256 threads): warp 0 streams K/V tiles with TMA (3 stages),
// warp 1 issues the MMAs from one thread, warp 2 owns the TMEM allocation,
// warps 4-7 are the softmax warpgroup: thread t owns query row t, so the row
// maximum and sum need no shuffles. S is double-buffered in TMEM so S_{j+1}
// runs while row statistics of tile j are formed; P goes to shared memory
// (128-byte swizzled, K-major) for the PV product. O is rescaled lazily: only
// when a row maximum grows by more than 2^8 (FlashAttention-style online
// softmax with a stale maximum; P stays <= 256). Partials use log2 units, as in
// attn.cuh, and finish through the same split combine / FlashBlock merge.
#pragma once

#include "attn.cuh"
#include "tc.cuh"

namespace fb {

constexpr int kTcStages = 3;
constexpr int kTcThreads = 256;
constexpr int kTcRows = 128;
constexpr int kTcProducer = 0, kTcMma = 1, kTcAlloc = 2, kTcSoft0 = 4;
constexpr uint32_t kTcCols = 256;  // S0 [0,64), S1 [64,128), O [128,256)
constexpr float kTcRescale = 8.f;  // log2 of the largest P value allowed before rescaling O

struct TcSmem {
  static constexpr int kHalf = kTcRows * 128;             // one 64-channel half of Q
  static constexpr int kQBytes = 2 * kHalf;               // 32 KB
  static constexpr int kKVHalf = kTK * 128;               // one 64-channel half of a K or V tile
  static constexpr int kTile = 2 * kKVHalf;               // K or V tile: 16 KB
  static constexpr int kStage = 2 * kTile;                // K + V: 32 KB
  static constexpr int kP = kTcRows * 128;                // P: 128 rows x 64 keys bf16
  static constexpr int kBytes = 1024 + kQBytes + kTcStages * kStage + 2 * kP;
};

__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV) {
  constexpr int D = 128;
  using S = TcSmem;
  __shared__ __align__(8) uint64_t full_bar[kTcStages];
  __shared__ __align__(8) uint64_t empty_bar[kTcStages];
  __shared__ __align__(8) uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  __shared__ __align__(8) uint64_t q_ready, mma_done;
  __shared__ int meta[kTcStages][kMaxChunks];
  __shared__ int meta_full[kTcStages];
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_base_sh;
  extern __shared__ uint8_t dyn_smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x % a.n_row_tiles;
  const int split = blockIdx.x / a.n_row_tiles;
  const int hk = blockIdx.y, b = blockIdx.z;
  if (!cta_selected(a, b, hk)) return;
  const int n_tiles = n_tiles_of(a, b, hk);
  const int tile0 = split * a.tiles_per_split;
  const int n_it = max(0, min(a.tiles_per_split, n_tiles - tile0));
  const int n_chunks = kTK / a.chunk;

  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* base_ptr = dyn_smem + (base - smem_u32(dyn_smem));
  const uint32_t sQ = base;
  const uint32_t sKV0 = base + S::kQBytes;
  const uint32_t sP0 = sKV0 + kTcStages * S::kStage;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(&q_ready, 4);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTcAlloc) tmem_alloc(&tmem_base_sh, kTcCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kTcProducer) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int st = it % kTcStages;
        const uint32_t ph = (it / kTcStages) & 1;
        if (!mbar_wait(&empty_bar[st], ph ^ 1, &abort_flag)) break;
        long long slots[kMaxChunks];
        int all_full = 1;
        for (int c = 0; c < n_chunks; ++c) {
          int valid;
          chunk_slot(a, b, hk, tile0 + it, c, slots[c], valid);
          meta[st][c] = valid;
          all_full &= (valid == a.chunk);
        }
        meta_full[st] = all_full;
        mbar_arrive_expect_tx(&full_bar[st], S::kStage);
        uint8_t* sk = base_ptr + (sKV0 - base) + st * S::kStage;
        uint8_t* sv = sk + S::kTile;
        for (int c = 0; c < n_chunks; ++c) {
          const int z = (int)slots[c];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sk + hf * S::kKVHalf + c * a.chunk * 128, &tmK, hf * 64, hk, z,
                        &full_bar[st]);
            tma_load_3d(sv + hf * S::kKVHalf + c * a.chunk * 128, &tmV, hf * 64, hk, z,
                        &full_bar[st]);
          }
        }
        ++issued;
      }
      if (abort_flag) {
        const long long t0 = clock64();
        for (int it = max(0, issued - kTcStages); it < issued; ++it) {
          const int st = it % kTcStages;
          const uint32_t ph = (it / kTcStages) & 1;
          while (!mbar_try_wait(&full_bar[st], ph) && clock64() - t0 < kWaitBudgetCycles) {
          }
        }
      }
    }
  } else if (warp == kTcMma) {
    // ------------------------------ MMA issuer -------------------------------
    if (lane == 0 && n_it > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTcRows, kTK, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kTcRows, D, 0, 1);
      bool ok = mbar_wait(&q_ready, 0, &abort_flag);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int st = j % kTcStages;
        if (!mbar_wait(&full_bar[st], (j / kTcStages) & 1, &abort_flag)) return false;
        const int sb = j & 1;
        if (j >= 2 && !mbar_wait(&s_free[sb], ((j - 2) >> 1) & 1, &abort_flag)) return false;
        tc_fence_after();
        const uint32_t sK = sKV0 + st * S::kStage;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 channels = 32 bytes along the swizzled row
          const uint64_t ad = smem_desc_sw128(sQ + (kk >> 2) * S::kHalf + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + (kk >> 2) * S::kKVHalf + off, 16, 1024);
          tc_mma(tmem + sb * kTK, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_it; ++j) {
        if (j + 1 < n_it && !issue_s(j + 1)) break;
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, &abort_flag)) break;
        tc_fence_after();
        const int st = j % kTcStages;
        const uint32_t sV = sKV0 + st * S::kStage + S::kTile;
        const uint32_t sP = sP0 + (j & 1) * S::kP;
#pragma unroll
        for (int ks = 0; ks < kTK / 16; ++ks) {
          const uint64_t ad = smem_desc_sw128(sP + ks * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sV + ks * 16 * 128, S::kKVHalf, 1024);
          tc_mma(tmem + 2 * kTK, ad, bd, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[j & 1]);
        tc_commit(&empty_bar[st]);
      }
      // every MMA of this CTA has completed before TMEM is released
      tc_commit(&mma_done);
      const long long t0 = clock64();
      while (!mbar_try_wait(&mma_done, 0) && clock64() - t0 < kWaitBudgetCycles) {
      }
    }
  } else if (warp >= kTcSoft0) {
    // --------------------------- softmax warpgroup ----------------------------
    const int trow = (warp - kTcSoft0) * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
    const int r = rt * kTcRows + trow;
    {  // this row of Q into shared memory, 128-byte swizzled, K-major
      const uint4* src = nullptr;
      if (r < a.R) {
        int i, h;
        row_of(a, b, hk, r, i, h);
        src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                             (((long long)b * a.B + i) * a.Hq + h) * D);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = src ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        const int hf = c >> 3, cc = c & 7;
        uint8_t* dst = base_ptr + hf * S::kHalf + (trow >> 3) * 1024 + (trow & 7) * 128 +
                       ((cc ^ (trow & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }
    float m_used = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < n_it; ++j) {
      mbar_wait(&s_full[j & 1], (j >> 1) & 1, &abort_flag);
      // lanes leave their waits at different times; the TMEM loads below are
      // warp-collective (.sync.aligned) and need the warp converged
      __syncwarp();
      tc_fence_after();
      float sv[kTK];
      {
        float lo[32], hi[32];
        tmem_ld32(tmem + t_lane + (j & 1) * kTK, lo);
        tmem_ld32(tmem + t_lane + (j & 1) * kTK + 32, hi);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          sv[k] = lo[k];
          sv[32 + k] = hi[k];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[j & 1]);
      const int st = j % kTcStages;
      // acquire the producer's tile metadata through the TMA barrier itself
      // (its phase for tile j is complete: S_j was computed from that stage)
      mbar_wait(&full_bar[st], (j / kTcStages) & 1, &abort_flag);
      const bool tile_full = meta_full[st] != 0;
      const int chunk = a.chunk;
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < kTK; ++k) {
        float x = sv[k] * a.scale_log2;
        if (!tile_full) {
          const int ci = k / chunk;
          if (k - ci * chunk >= meta[st][ci]) x = -INFINITY;
        }
        sv[k] = x;
        mx = fmaxf(mx, x);
      }
      if (!tile_full && trow < kTK) {
        // the V row of a key outside the key set may hold any bits: zero it
        const int ci = trow / chunk;
        if (trow - ci * chunk >= meta[st][ci]) {
          uint8_t* vrow = base_ptr + (sKV0 - base) + st * S::kStage + S::kTile +
                          (trow >> 3) * 1024 + (trow & 7) * 128;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              *reinterpret_cast<uint4*>(vrow + hf * S::kKVHalf + (cc << 4)) =
                  make_uint4(0u, 0u, 0u, 0u);
        }
      }
      const float m_new = fmaxf(m_used, mx);
      // Rescale when this row's maximum grew by more than 2^8. The TMEM loads
      // and stores are warp-collective (.sync.aligned), so the decision is
      // taken per warp: if any row of the warp needs it, every lane rescales,
      // the others by exactly 1.
      const bool need = m_new > m_used + kTcRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;  // 0 if nothing accumulated
        if (j > 0) {
          mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, &abort_flag);
          __syncwarp();
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tmem + t_lane + 2 * kTK + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= alpha;
            tmem_st32(tmem + t_lane + 2 * kTK + c * 32, o);
          }
          tmem_wait_st();
        }
        if (need) {
          l_sum *= alpha;
          m_used = m_new;
        }
      }
      const float bse = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[kTK / 2];
#pragma unroll
      for (int k = 0; k < kTK; k += 2) {
        const float p0 = fast_exp2(sv[k] - bse), p1 = fast_exp2(sv[k + 1] - bse);
        l_sum += p0 + p1;
        pk[k >> 1] = pack_bf16(p0, p1);
      }
      if (j >= 2) mbar_wait(&pv_done[j & 1], ((j - 2) >> 1) & 1, &abort_flag);  // P buffer free
      __syncwarp();
      uint8_t* prow = base_ptr + (sP0 - base) + (j & 1) * S::kP + (trow >> 3) * 1024 +
                      (trow & 7) * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4*>(prow + ((cc ^ (trow & 7)) << 4)) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
    }
    // ---------------------------- epilogue (one row per thread) -------------------
    if (n_it > 0) {
      mbar_wait(&pv_done[(n_it - 1) & 1], ((n_it - 1) >> 1) & 1, &abort_flag);
      __syncwarp();
      tc_fence_after();
    }
    const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
    const float lse2 = l_sum > 0.f ? m_used + log2f(l_sum) : -INFINITY;
    // merge partner of the final row (FlashBlock merge), read before any store
    long long row = -1;
    bool write = r < a.R;
    float wn = 1.f, wo = 0.f, Lfin = lse2 * kLn2;
    if (write && a.n_splits <= 1) {
      int i, h;
      row_of(a, b, hk, r, i, h);
      write = row_selected(a, b, h);
      row = ((long long)b * a.B + i) * a.Hq + h;
      if (write && a.mrg_a) {
        const float Lo = a.mrg_l[row];
        const float m = fmaxf(Lo, Lfin);
        if (m == -INFINITY) {
          wn = 0.f;
          Lfin = -INFINITY;
        } else {
          const float eo = expf(Lo - m), en = expf(Lfin - m);
          const float s = 1.f / (eo + en);
          wn = en * s;
          wo = eo * s;
          Lfin = m + logf(eo + en);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      __syncwarp();  // the stores of the previous chunk diverge by row
      if (n_it > 0) {
        tmem_ld32(tmem + t_lane + 2 * kTK + c * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0.f;
      }
      if (!write) continue;
      if (a.n_splits > 1) {
        const long long pidx = (((long long)split * a.batch + b) * a.Hkv + hk) * a.R + r;
        float4* dst = reinterpret_cast<float4*>(a.o_part + pidx * D + c * 32);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                               o[4 * k + 3] * inv);
      } else {
        float4* dst = reinterpret_cast<float4*>(a.a_out + row * D + c * 32);
        const float4* old = a.mrg_a ? reinterpret_cast<const float4*>(a.mrg_a + row * D + c * 32)
                                    : nullptr;
        float4* prv = a.a_prev ? reinterpret_cast<float4*>(a.a_prev + row * D + c * 32) : nullptr;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float4 v = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                 o[4 * k + 3] * inv);
          if (a.mrg_a) {
            const float4 u = wo > 0.f ? old[k] : make_float4(0.f, 0.f, 0.f, 0.f);
            v = make_float4(wn * v.x + wo * u.x, wn * v.y + wo * u.y, wn * v.z + wo * u.z,
                            wn * v.w + wo * u.w);
            if (wn == 0.f && wo == 0.f) v = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          if (prv) prv[k] = dst[k];
          dst[k] = v;
        }
      }
    }
    if (write) {
      if (a.n_splits > 1) {
        const long long pidx = (((long long)split * a.batch + b) * a.Hkv + hk) * a.R + r;
        a.lse_part[pidx] = lse2;
      } else {
        a.l_out[row] = Lfin;
      }
    }
  }
  // ------------------------------- teardown ---------------------------------
  // Warps 0 and 1 ran their loops on lane 0 alone: reconverge every warp before
  // the block-wide barrier (an aligned barrier reached by a divergent warp is
  // undefined and can complete without the busy lane, letting TMEM be freed
  // under in-flight MMAs and leaving that lane waiting forever).
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTcAlloc) tmem_free(tmem, kTcCols);
}

}  // namespace fb
