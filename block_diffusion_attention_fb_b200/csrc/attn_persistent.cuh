// Persistent split-KV attention partial for R <= 64 stacked rows per kv head
// (the dLLM prefix, LoSA's dense first step and its sparse gather), bf16.
//
// Work = the kTK-key tiles of every (sequence b, kv head hk) group laid end to
// end; CTA c of n (two per SM) streams tiles [c*T/n, (c+1)*T/n), so each SM
// moves the same number of bytes whatever the prefix lengths, and the TMA
// pipeline of a CTA runs on across group boundaries. A group covered by one
// CTA is written out directly; a group spread over several CTAs leaves one
// partial per CTA (at most two per CTA: its first and its last group) and the
// CTA that takes the group's last ticket merges them by the log-space rule
// (FlashBlock technical summary §2, merge equation) and writes the rows.
// Math per tile as in attn_bf16_kernel: mma.sync bf16 m16n8k16, fp32 online
// softmax in the exp2 domain, RG row groups x KS key slices over 4 warps.
#pragma once

#include "attn.cuh"

namespace fb {

constexpr int kStagesP = 2;
constexpr int kMaxGroupsP = 1024;
constexpr int kPersistCtasPerSm = 2;

template <int D>
struct PersistSmem {
  static constexpr int kStage = Bf16Smem<D>::kStageBytes;
  static constexpr int kRedStride = D + 4;
  // softmax states of the warps with key slice > 0 (at most three warps)
  static constexpr int kRedBytes = 3 * 16 * kRedStride * 4 + 2 * 3 * 16 * 4;
  static constexpr int kPrefixBytes = (kMaxGroupsP + 1) * 4;
  static constexpr int kBytes = 1024 + kStagesP * kStage + kRedBytes + kPrefixBytes;
};

template <int D, int RG>
__global__ void __launch_bounds__(kAttnThreads, kPersistCtasPerSm)
    attn_bf16_persistent(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV) {
  using S = Bf16Smem<D>;
  using P = PersistSmem<D>;
  constexpr int KS = kNWC / RG;
  constexpr int KW = kTK / KS;
  constexpr int SUB = KW < 32 ? KW : 32;
  constexpr int NT = SUB / 8;
  constexpr int KD = D / 16;
  constexpr int NV = D / 32;

  __shared__ __align__(8) uint64_t full_bar[kStagesP];
  __shared__ __align__(8) uint64_t empty_bar[kStagesP];
  __shared__ int meta[kStagesP][kMaxChunks];
  __shared__ int meta_full[kStagesP];
  __shared__ int abort_flag;
  __shared__ int s_last;
  extern __shared__ uint8_t dyn_smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* base_ptr = dyn_smem + (base - smem_u32(dyn_smem));
  float* red = reinterpret_cast<float*>(base_ptr + kStagesP * P::kStage);
  int* prefix = reinterpret_cast<int*>(base_ptr + kStagesP * P::kStage + P::kRedBytes);

  // ---- tile counts of every group and their prefix sums (every CTA) ----
  const int n_groups = a.batch * a.Hkv;
  for (int g = tid; g < n_groups; g += blockDim.x) {
    const int b = g / a.Hkv, hk = g - (g / a.Hkv) * a.Hkv;
    prefix[g + 1] = cta_selected(a, b, hk) ? n_tiles_of(a, b, hk) : 0;
  }
  if (tid == 0) {
    prefix[0] = 0;
    for (int s = 0; s < kStagesP; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kNWC);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of prefix[1..n_groups] by one warp
    const int per = (n_groups + 31) / 32;
    const int g0 = lane * per, g1 = min(n_groups, g0 + per);
    int run = 0;
    for (int g = g0; g < g1; ++g) {
      run += prefix[g + 1];
      prefix[g + 1] = run;
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - run;
    for (int g = g0; g < g1; ++g) prefix[g + 1] += excl;
  }
  __syncthreads();
  const long long T = prefix[n_groups];
  const int n_cta = gridDim.x, c = blockIdx.x;

  // Selected groups with no key at all (an empty prefix): A = 0, L = -inf (or
  // just the merge partner), written by CTA g mod n_cta.
  if (warp < kNWC) {
    for (int g = c; g < n_groups; g += n_cta) {
      if (prefix[g + 1] != prefix[g]) continue;
      const int b = g / a.Hkv, hk = g - (g / a.Hkv) * a.Hkv;
      if (!cta_selected(a, b, hk)) continue;
      float zero[NV];
#pragma unroll
      for (int j = 0; j < NV; ++j) zero[j] = 0.f;
      for (int r = warp; r < a.R; r += kNWC)
        write_final<NV>(a, b, hk, r, zero, lane * NV, 1, -INFINITY, lane == 0);
    }
  }

  const long long t0 = (long long)c * T / n_cta, t1 = (long long)(c + 1) * T / n_cta;
  if (t0 >= t1) return;
  auto tile_start_of = [&](int cc) { return (long long)cc * T / n_cta; };
  auto locate = [&](long long t) {  // group with prefix[g] <= t < prefix[g+1]
    int lo = 0, hi = n_groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    while (prefix[lo + 1] <= t) ++lo;
    return lo;
  };
  const int n_chunks = kTK / a.chunk;

  if (warp == kNWC) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int g = locate(t0);
      int local = (int)(t0 - prefix[g]);
      long long issued = 0;
      for (long long t = t0; t < t1; ++t) {
        const int it = (int)(t - t0);
        const int st = it % kStagesP;
        const uint32_t ph = (it / kStagesP) & 1;
        if (!mbar_wait(&empty_bar[st], ph ^ 1, &abort_flag)) break;
        const int b = g / a.Hkv, hk = g - (g / a.Hkv) * a.Hkv;
        long long slots[kMaxChunks];
        int all_full = 1;
        for (int ci = 0; ci < n_chunks; ++ci) {
          int valid;
          chunk_slot(a, b, hk, local, ci, slots[ci], valid);
          meta[st][ci] = valid;
          all_full &= (valid == a.chunk);
        }
        meta_full[st] = all_full;
        mbar_arrive_expect_tx(&full_bar[st], S::kStageBytes);
        uint8_t* sk = base_ptr + st * S::kStageBytes;
        uint8_t* sv = sk + S::kTileBytes;
        for (int ci = 0; ci < n_chunks; ++ci) {
          const int z = (int)slots[ci];
#pragma unroll
          for (int hf = 0; hf < S::kHalves; ++hf) {
            tma_load_3d(sk + hf * S::kHalfBytes + ci * a.chunk * 128, &tmK, hf * 64, hk, z,
                        &full_bar[st]);
            tma_load_3d(sv + hf * S::kHalfBytes + ci * a.chunk * 128, &tmV, hf * 64, hk, z,
                        &full_bar[st]);
          }
        }
        ++issued;
        if (++local == prefix[g + 1] - prefix[g]) {
          local = 0;
          do {
            ++g;
          } while (g < n_groups && prefix[g + 1] == prefix[g]);
        }
      }
      if (abort_flag) {
        const long long tw = clock64();
        for (long long it = issued > kStagesP ? issued - kStagesP : 0; it < issued; ++it) {
          const int st = (int)(it % kStagesP);
          const uint32_t ph = (uint32_t)((it / kStagesP) & 1);
          while (!mbar_try_wait(&full_bar[st], ph) && clock64() - tw < kWaitBudgetCycles) {
          }
        }
      }
    }
    return;
  }

  // ------------------------------ consumers -------------------------------
  const int rg = warp % RG, ks = warp / RG;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q);

  uint32_t qa[KD][4];
  float o[D / 8][4];
  float m_r[2], l_r[2];

  int g = locate(t0);
  int local = (int)(t0 - prefix[g]);
  long long seg_t0 = t0;
  for (long long t = t0; t < t1; ++t) {
    const int it = (int)(t - t0);
    const int T_g = prefix[g + 1] - prefix[g];
    const int b = g / a.Hkv, hk = g - (g / a.Hkv) * a.Hkv;
    if (t == t0 || local == 0) {
      // new segment: the group's query rows, a fresh softmax state
      seg_t0 = t;
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = rg * 16 + g8 + hr * 8;
        const __nv_bfloat16* rowp = nullptr;
        if (r < a.R) {
          int i, h;
          row_of(a, b, hk, r, i, h);
          rowp = qb + (((long long)b * a.B + i) * a.Hq + h) * D;
        }
#pragma unroll
        for (int kk = 0; kk < KD; ++kk) {
          const int col = kk * 16 + 2 * t4;
          qa[kk][hr] = rowp ? *reinterpret_cast<const uint32_t*>(rowp + col) : 0u;
          qa[kk][hr + 2] = rowp ? *reinterpret_cast<const uint32_t*>(rowp + col + 8) : 0u;
        }
      }
#pragma unroll
      for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      m_r[0] = m_r[1] = -INFINITY;
      l_r[0] = l_r[1] = 0.f;
    }
    const int st = it % kStagesP;
    const uint32_t ph = (it / kStagesP) & 1;
    // a timed-out wait sets the error word and abort flag; the loop keeps its
    // shape so every consumer warp still meets the named barriers below
    mbar_wait(&full_bar[st], ph, &abort_flag);
    const uint32_t sK = base + st * S::kStageBytes;
    const uint32_t sV = sK + S::kTileBytes;
    const bool tile_full = meta_full[st] != 0;
    const int chunk = a.chunk;
    bool wrote_smem = false;
#pragma unroll
    for (int sub = 0; sub < KW / SUB; ++sub) {
      const int kb = ks * KW + sub * SUB;
      float s[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const int key = kb + np * 16 + (mi >> 1) * 8 + r8;
          const int ch = 2 * kk + (mi & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sK + (ch >> 3) * S::kHalfBytes + key * 128 + (((ch & 7) ^ (key & 7)) << 4), b0,
                  b1, b2, b3);
          mma_bf16(s[2 * np], qa[kk], b0, b1);
          mma_bf16(s[2 * np + 1], qa[kk], b2, b3);
        }
      }
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
            const int cix = key / chunk;
            if (key - cix * chunk >= meta[st][cix]) s[n][e] = -INFINITY;
          }
        for (int idx = lane; idx < SUB * (D / 8); idx += 32) {
          const int kr = idx / (D / 8), ch = idx % (D / 8);
          const int key = kb + kr;
          const int cix = key / chunk;
          if (key - cix * chunk >= meta[st][cix]) {
            uint8_t* p = base_ptr + (sV - base) + (ch >> 3) * S::kHalfBytes + key * 128 +
                         (((ch & 7) ^ (key & 7)) << 4);
            *reinterpret_cast<uint4*>(p) = make_uint4(0u, 0u, 0u, 0u);
            wrote_smem = true;
          }
        }
        __syncwarp();
      }
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
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s[n][e] = fast_exp2(s[n][e] - bse[e >> 1]);
          rs[e >> 1] += s[n][e];
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
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + (ch >> 3) * S::kHalfBytes + key * 128 + (((ch & 7) ^ (key & 7)) << 4),
                    b0, b1, b2, b3);
          mma_bf16(o[2 * dp], pa, b0, b1);
          mma_bf16(o[2 * dp + 1], pa, b2, b3);
        }
      }
    }
    if (wrote_smem) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);

    const bool seg_end = (t == t1 - 1) || (local == T_g - 1);
    if (seg_end) {
      // ------------- epilogue of this CTA's segment of group g -------------
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
        l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
      }
      if (KS > 1) {
        float* rO = red;
        float* rM = red + 3 * 16 * P::kRedStride;
        float* rL = rM + 3 * 16;
        if (ks > 0) {
          const int slot = (ks - 1) * RG + rg;  // < 3 since RG * KS == 4
#pragma unroll
          for (int n = 0; n < D / 8; ++n) {
            const int col = n * 8 + 2 * t4;
            *reinterpret_cast<float2*>(&rO[(slot * 16 + g8) * P::kRedStride + col]) =
                make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2*>(&rO[(slot * 16 + g8 + 8) * P::kRedStride + col]) =
                make_float2(o[n][2], o[n][3]);
          }
          if (t4 == 0) {
            rM[slot * 16 + g8] = m_r[0];
            rM[slot * 16 + g8 + 8] = m_r[1];
            rL[slot * 16 + g8] = l_r[0];
            rL[slot * 16 + g8 + 8] = l_r[1];
          }
        }
        named_bar_sync(1, kNWC * 32);
        if (ks == 0) {
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            float M = m_r[hr];
#pragma unroll
            for (int k = 1; k < KS; ++k) M = fmaxf(M, rM[((k - 1) * RG + rg) * 16 + g8 + hr * 8]);
            const float bm = (M == -INFINITY) ? 0.f : M;
            const float w0 = fast_exp2(m_r[hr] - bm);
            float lsum = l_r[hr] * w0;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
              o[n][2 * hr] *= w0;
              o[n][2 * hr + 1] *= w0;
            }
#pragma unroll
            for (int k = 1; k < KS; ++k) {
              const int slot = (k - 1) * RG + rg;
              const float wk = fast_exp2(rM[slot * 16 + g8 + hr * 8] - bm);
              lsum += wk * rL[slot * 16 + g8 + hr * 8];
#pragma unroll
              for (int n = 0; n < D / 8; ++n) {
                const float2 v = *reinterpret_cast<const float2*>(
                    &rO[(slot * 16 + g8 + hr * 8) * P::kRedStride + n * 8 + 2 * t4]);
                o[n][2 * hr] += wk * v.x;
                o[n][2 * hr + 1] += wk * v.y;
              }
            }
            m_r[hr] = M;
            l_r[hr] = lsum;
          }
        }
        named_bar_sync(1, kNWC * 32);  // merge area free again
      }
      const bool whole_group = (seg_t0 == prefix[g]) && (local == T_g - 1);
      const int slot_idx = (seg_t0 == t0) ? 0 : 1;
      if (ks == 0) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = rg * 16 + g8 + hr * 8;
          if (r >= a.R) continue;
          const float inv = l_r[hr] > 0.f ? 1.f / l_r[hr] : 0.f;
          const float lse2 = l_r[hr] > 0.f ? m_r[hr] + log2f(l_r[hr]) : -INFINITY;
          if (whole_group) {
            int i, h;
            row_of(a, b, hk, r, i, h);
            if (!row_selected(a, b, h)) continue;
            const long long row = ((long long)b * a.B + i) * a.Hq + h;
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
                const float sc = 1.f / (eo + en);
                wn = en * sc;
                wo = eo * sc;
                L = m + logf(eo + en);
              }
            }
            float* dst = a.a_out + row * D;
            const float* old = a.mrg_a ? a.mrg_a + row * D : nullptr;
            float* prv = a.a_prev ? a.a_prev + row * D : nullptr;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
              const int col = n * 8 + 2 * t4;
              float2 v = make_float2(wn * o[n][2 * hr] * inv, wn * o[n][2 * hr + 1] * inv);
              if (old && wo > 0.f) {
                const float2 u = *reinterpret_cast<const float2*>(old + col);
                v.x += wo * u.x;
                v.y += wo * u.y;
              }
              if (prv)
                *reinterpret_cast<float2*>(prv + col) = *reinterpret_cast<const float2*>(dst + col);
              *reinterpret_cast<float2*>(dst + col) = v;
            }
            if (t4 == 0) a.l_out[row] = L;
          } else {
            const long long pidx = ((long long)c * 2 + slot_idx) * a.R + r;
            float* dst = a.o_part + pidx * D;
#pragma unroll
            for (int n = 0; n < D / 8; ++n)
              *reinterpret_cast<float2*>(dst + n * 8 + 2 * t4) =
                  make_float2(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
            if (t4 == 0) a.lse_part[pidx] = lse2;
          }
        }
      }
      if (!whole_group) {
        // the CTA that brings the group's last partial merges all of them
        __threadfence();
        int c_a = (int)((long long)prefix[g] * n_cta / T);
        while (c_a + 1 < n_cta && tile_start_of(c_a + 1) <= prefix[g]) ++c_a;
        while (c_a > 0 && tile_start_of(c_a) > prefix[g]) --c_a;
        const long long last_tile = prefix[g + 1] - 1;
        int c_b = (int)(last_tile * n_cta / T);
        while (c_b + 1 < n_cta && tile_start_of(c_b + 1) <= last_tile) ++c_b;
        while (c_b > 0 && tile_start_of(c_b) > last_tile) --c_b;
        // CTAs with an empty tile range (more CTAs than tiles) contribute nothing
        int n_contrib = 0;
        for (int cc = c_a; cc <= c_b; ++cc) n_contrib += tile_start_of(cc) < tile_start_of(cc + 1);
        named_bar_sync(1, kNWC * 32);
        if (tid == 0) s_last = atomicAdd(&a.tickets[g], 1) == n_contrib - 1;
        named_bar_sync(1, kNWC * 32);
        if (s_last) {
          __threadfence();
          for (int r = warp; r < a.R; r += kNWC) {
            // one partial per lane (c_b - c_a < 32 here: n_cta <= 2 * SMs over >= 1 group)
            float M = -INFINITY;
            for (int cc = c_a + lane; cc <= c_b; cc += 32) {
              if (tile_start_of(cc) >= tile_start_of(cc + 1)) continue;
              const int sl = (cc == c_a && prefix[g] > tile_start_of(c_a)) ? 1 : 0;
              M = fmaxf(M, __ldcg(a.lse_part + ((long long)cc * 2 + sl) * a.R + r));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            const float bm = (M == -INFINITY) ? 0.f : M;
            float acc[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) acc[j] = 0.f;
            float wsum = 0.f;
            const long long pidx_a =
                ((long long)c_a * 2 + (prefix[g] > tile_start_of(c_a) ? 1 : 0)) * a.R + r;
            for (int cb = c_a; cb <= c_b; cb += 32) {
              // lane k: the (cb + k)-th CTA's partial and weight; empty CTAs get
              // weight 0 and point at a written partial, so every load below is
              // issued unconditionally and they overlap
              const int cc = cb + lane;
              long long pidx = pidx_a;
              float w = 0.f;
              if (cc <= c_b && tile_start_of(cc) < tile_start_of(cc + 1)) {
                const int sl = (cc == c_a && prefix[g] > tile_start_of(c_a)) ? 1 : 0;
                pidx = ((long long)cc * 2 + sl) * a.R + r;
                const float l = __ldcg(a.lse_part + pidx);
                w = l == -INFINITY ? 0.f : fast_exp2(l - bm);
              }
              const int n = min(32, c_b - cb + 1);
#pragma unroll 8
              for (int k = 0; k < n; ++k) {
                const float wk = __shfl_sync(0xffffffffu, w, k);
                const long long pk = __shfl_sync(0xffffffffu, pidx, k);
                wsum += wk;
                const float* src = a.o_part + pk * D + lane * NV;
#pragma unroll
                for (int j = 0; j < NV; ++j) acc[j] += wk * __ldcg(src + j);
              }
            }
            const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
            for (int j = 0; j < NV; ++j) acc[j] *= inv;
            const float lse2 = wsum > 0.f ? bm + log2f(wsum) : -INFINITY;
            write_final<NV>(a, b, hk, r, acc, lane * NV, 1, lse2, lane == 0);
          }
        }
      }
    }
    if (++local == T_g) {
      local = 0;
      do {
        ++g;
      } while (g < n_groups && prefix[g + 1] == prefix[g]);
    }
  }
}

}  // namespace fb
