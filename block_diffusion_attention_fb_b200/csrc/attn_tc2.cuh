// Attention partial on the 5th-generation tensor cores (tcgen05), head_dim 128,
// for key sets read by many stacked query rows (GQA groups, video blocks).
//
// Same outputs as attn_bf16_kernel (split partials or final rows, optional
// FlashBlock merge); the partial of one query row over its key set follows the
// FlashBlock technical summary, §2 "Core mechanism". The design is set by the
// two per-SM limits of this shape: the tensor core (S = QK^T and O += PV cost
// 512 flops per score) and the exponential unit (one 2^x per score), which at
// head_dim 128 run at the same rate. Keeping both busy takes two independent
// softmax streams, so a CTA owns TWO 128-row Q tiles (A and B, 256 stacked rows)
// that share every K/V tile read from HBM:
//
//   warp 0      TMA producer: 128-key K and V tiles (32 KB each) into a ring of
//               5 slots, loaded in the order K_0 V_0 K_1 V_1 ...: K_j is freed
//               once both S MMAs have read it, V_j once both PV MMAs have, so
//               up to three tiles are in flight while two are in use
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_X = Q_X K_j^T        (M 128, N 128 keys, K 128) -> TMEM
//                 O_X += P_X V_j         (M 128, N 128 channels, K 128 keys),
//                                         P_X read from TMEM (no shared-memory trip)
//               issued in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the
//               tensor core works on one tile while the other tile's softmax runs
//   warps 4-7   softmax of tile A; warps 8-11: tile B. Thread t owns row t of
//               its tile (TMEM lane t): row maximum and sum need no shuffles.
//               S_X is loaded into registers, P_X = 2^(S - m) is written back
//               as bf16 over the first 64 columns of S_X, and O_X is rescaled
//               lazily in TMEM (only when the row maximum grows by more than
//               2^8, so P <= 256).
// TMEM: S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512) columns.
// Ordering: tcgen05.mma operations of one thread run in issue order, so
// S_X(j+1), issued after PV_X(j), overwrites P_X(j) only once PV_X(j) has read
// it; the completion of S_X(j) (its commit barrier) also covers PV_X(j-1), so
// the softmax may rescale O_X then.
// Partials are kept in log2 units, as in attn.cuh, and finish through the same
// split combine / FlashBlock merge.
#pragma once

#include "attn.cuh"
#include "tc.cuh"

namespace fb {

constexpr int kT2Keys = 128;  // keys per K/V tile (two 64-key metadata sub-tiles)
constexpr int kT2Slots = 5;   // ring of 32 KB K or V tiles
constexpr int kT2Meta = 4;    // ring of tile metadata entries
constexpr int kT2Threads = 384;
constexpr int kT2TileRows = 128;  // rows per Q tile; a CTA owns two
constexpr int kT2Rows = 2 * kT2TileRows;
constexpr int kT2Producer = 0, kT2Mma = 1, kT2SoftA = 4, kT2SoftB = 8;
constexpr uint32_t kT2Cols = 512;
constexpr float kT2Rescale = 8.f;  // log2 of the largest P value before O is rescaled
constexpr int kT2LowRegs = 72, kT2HighRegs = 216;
static_assert(4 * 32 * kT2LowRegs + 8 * 32 * kT2HighRegs <= kT2Threads * 168,
              "register split exceeds the launch's registers");

struct Tc2Smem {
  static constexpr int kQHalf = kT2TileRows * 128;  // 128 rows x 64 channels bf16
  static constexpr int kQTile = 2 * kQHalf;         // 32 KB
  static constexpr int kKVHalf = kT2Keys * 128;     // 128 keys x 64 channels
  static constexpr int kKVTile = 2 * kKVHalf;       // one K or V tile: 32 KB
  static constexpr int kBytes = 1024 + 2 * kQTile + kT2Slots * kKVTile;
};

__global__ void __launch_bounds__(kT2Threads, 1)
    attn_tc2_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV) {
  grid_dependency_wait();  // launched as a programmatic dependent
  allow_dependent_launch();
  constexpr int D = 128;
  using S = Tc2Smem;
  __shared__ __align__(8) uint64_t full_bar[kT2Slots];
  __shared__ __align__(8) uint64_t empty_bar[kT2Slots];
  __shared__ __align__(8) uint64_t meta_bar[kT2Meta];
  __shared__ __align__(8) uint64_t s_full[2], p_full[2], o_done[2];
  __shared__ __align__(8) uint64_t q_ready, mma_done;
  // Metadata of tile j lives in entry j % 4. The producer rewrites an entry
  // for tile j + 4 only after V_{j+1}'s slot was freed, i.e. after both
  // softmax warpgroups finished tile j + 1, so a reader never sees its entry's
  // barrier advance twice.
  __shared__ int meta[kT2Meta][2 * kMaxChunks];
  __shared__ int meta_full[kT2Meta];
  // chunk slots / valid counts of upcoming tiles, filled by the producer warp
  __shared__ int ring_slot[kSlotRing][2 * kMaxChunks];
  __shared__ int ring_valid[kSlotRing][2 * kMaxChunks];
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_base_sh;
  extern __shared__ uint8_t dyn_smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x % a.n_row_tiles;
  const int split = blockIdx.x / a.n_row_tiles;
  const int hk = blockIdx.y, b = blockIdx.z;
  if (!cta_selected(a, b, hk)) return;
  const int Rb = rows_of(a, b);  // stacked rows of this sequence
  if (rt * kT2Rows >= Rb) return;
  // key range of this split in 64-key sub-tiles (an even number per split)
  const int n64_all = n_tiles_of(a, b, hk);
  const int tps = split_tiles(a, n64_all, true);
  const int n64 = max(0, min(tps, n64_all - split * tps));
  const int tile0 = split * tps;
  const int n_it = (n64 + 1) >> 1;  // 128-key tiles
  const int n_chunks = kTK / a.chunk;  // metadata chunks per 64-key sub-tile
  const bool has_b = Rb - rt * kT2Rows > kT2TileRows;

  const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* base_ptr = dyn_smem + (base - smem_u32(dyn_smem));
  const uint32_t sQ0 = base;                    // Q_A, then Q_B
  const uint32_t sKV0 = base + 2 * S::kQTile;   // ring of K / V tile slots

  if (tid == 0) {
    for (int s = 0; s < kT2Slots; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < kT2Meta; ++s) mbar_init(&meta_bar[s], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(&q_ready, has_b ? 8 : 4);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kT2Mma) tmem_alloc(&tmem_base_sh, kT2Cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Register split (launch: 384 threads x 168 = 64512): warps 0-3 give theirs
  // down to 72 (9216), the softmax warps take 216 (8 warps: 55296); the sum,
  // 64512, fits, so the increase never waits for registers that cannot come.
  // Each role changes its budget inside its own branch, so the compiler knows
  // the budget of every region.
  if (warp == kT2Producer) {
    reg_dealloc<kT2LowRegs>();
    // ------------------------------ TMA producer ------------------------------
    // Lane 0 waits for free slots and issues the copies; all 32 lanes fetch the
    // chunk slots of the tile kSlotAhead tiles ahead (one chunk per lane, the
    // page-list / page-table reads of a tile in flight together) into a small
    // shared ring, so those reads overlap the copies of the tiles before it.
    constexpr int kC = 2 * kMaxChunks;
    const int nc2 = 2 * n_chunks;  // chunks per 128-key tile
    const GroupInfo gi = group_info(a, b, hk);
    auto fill = [&](int it) {      // tile `it` -> ring entry it % kSlotRing (all lanes)
      if (lane < nc2) {
        // chunk c covers keys [c * chunk, (c + 1) * chunk) of the 128-key tile; a
        // sub-tile past the split's range gives valid = 0 (a zero-filled box)
        const int sub = lane / n_chunks, cc = lane - sub * n_chunks;
        long long s_ = a.n_slots;
        int v_ = 0;
        if (2 * it + sub < n64) chunk_slot(a, gi, b, hk, tile0 + 2 * it + sub, cc, s_, v_);
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
    int issued = 0;  // loads issued (K_0 = 0, V_0 = 1, K_1 = 2, ...)
    for (int n = 0; n < 2 * n_it; ++n) {
      const int it = n >> 1, is_v = n & 1;
      // ring entry (it + kSlotAhead) % kSlotRing last served tile it - 1, whose
      // copies were issued in the previous iterations
      if (!is_v && it + kSlotAhead < n_it) fill(it + kSlotAhead);
      int ok = 1;
      if (lane == 0) {
        const int sl = n % kT2Slots;
        const int re = it % kSlotRing;
        ok = mbar_wait(&empty_bar[sl], ((n / kT2Slots) & 1) ^ 1, &abort_flag);
        if (ok) {
          if (!is_v) {
            const int me = it % kT2Meta;
            int all_full = 1;
#pragma unroll
            for (int c = 0; c < kC; ++c) {
              if (c < nc2) {
                meta[me][c] = ring_valid[re][c];
                all_full &= (ring_valid[re][c] == a.chunk);
              }
            }
            meta_full[me] = all_full;
            mbar_arrive(&meta_bar[me]);  // release: the entry is written
          }
          mbar_arrive_expect_tx(&full_bar[sl], S::kKVTile);
          uint8_t* dst = base_ptr + (sKV0 - base) + sl * S::kKVTile;
          const CUtensorMap* tm = is_v ? &tmV : &tmK;
#pragma unroll
          for (int c = 0; c < kC; ++c) {
            if (c < nc2) {
              const int z = ring_slot[re][c];
              tma_load_3d(dst + c * a.chunk * 128, tm, 0, hk, z, &full_bar[sl]);
              tma_load_3d(dst + S::kKVHalf + c * a.chunk * 128, tm, 64, hk, z, &full_bar[sl]);
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
      for (int n = max(0, issued - kT2Slots); n < issued; ++n) {
        while (!mbar_try_wait(&full_bar[n % kT2Slots], (n / kT2Slots) & 1) &&
               clock64() - t0 < kWaitBudgetCycles) {
        }
      }
    }
  } else if (warp == kT2Mma) {
    reg_dealloc<kT2LowRegs>();
    // ------------------------------ MMA issuer -------------------------------
    if (lane == 0 && n_it > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kT2TileRows, kT2Keys, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kT2TileRows, D, 0, 1);
      const int nx = has_b ? 2 : 1;
      bool ok = mbar_wait(&q_ready, 0, &abort_flag);
      tc_fence_after();
      auto slot_wait = [&](int n) {  // load n (K_j = 2j, V_j = 2j + 1) has landed
        const bool r_ = mbar_wait(&full_bar[n % kT2Slots], (n / kT2Slots) & 1, &abort_flag);
        tc_fence_after();
        return r_;
      };
      auto issue_s = [&](int x, int j) {
        const uint32_t sQ = sQ0 + x * S::kQTile;
        const uint32_t sK = sKV0 + ((2 * j) % kT2Slots) * S::kKVTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 channels = 32 bytes along a swizzled row
          const uint64_t ad = smem_desc_sw128(sQ + (kk >> 2) * S::kQHalf + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + (kk >> 2) * S::kKVHalf + off, 16, 1024);
          tc_mma(tmem + x * kT2Keys, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint32_t sV = sKV0 + ((2 * j + 1) % kT2Slots) * S::kKVTile;
#pragma unroll
        for (int ks = 0; ks < kT2Keys / 16; ++ks) {
          const uint64_t bd = smem_desc_sw128(sV + ks * 16 * 128, S::kKVHalf, 1024);
          tc_mma_ts(tmem + 2 * kT2Keys + x * D, tmem + x * kT2Keys + ks * 8, bd, idesc_o,
                    (j > 0 || ks > 0) ? 1u : 0u);
        }
      };
      if (ok) ok = slot_wait(0);
      if (ok) {
        for (int x = 0; x < nx; ++x) issue_s(x, 0);
        tc_commit(&empty_bar[0]);  // K_0 is free once both S MMAs have read it
      }
      for (int j = 0; ok && j < n_it; ++j) {
        const bool more = j + 1 < n_it;
        ok = slot_wait(2 * j + 1);  // V_j
        for (int x = 0; x < nx && ok; ++x) {
          ok = mbar_wait(&p_full[x], j & 1, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_pv(x, j);
          if (more) {
            if (x == 0 && !(ok = slot_wait(2 * j + 2))) break;  // K_{j+1}
            issue_s(x, j + 1);
          }
        }
        if (!ok) break;
        tc_commit(&empty_bar[(2 * j + 1) % kT2Slots]);      // V_j: both PV MMAs done
        if (more) tc_commit(&empty_bar[(2 * j + 2) % kT2Slots]);  // K_{j+1}: both S MMAs done
      }
      if (ok)
        for (int x = 0; x < nx; ++x) tc_commit(&o_done[x]);
      // every MMA of this CTA has completed before TMEM is released
      tc_commit(&mma_done);
      const long long t0 = clock64();
      while (!mbar_try_wait(&mma_done, 0) && clock64() - t0 < kWaitBudgetCycles) {
      }
    }
  } else if (warp < kT2SoftA) {
    reg_dealloc<kT2LowRegs>();  // idle warps
  } else if (warp < kT2SoftB || has_b) {
    reg_alloc<kT2HighRegs>();
    // --------------------------- softmax warpgroups ----------------------------
    const int x = warp >= kT2SoftB ? 1 : 0;
    const int trow = (warp & 3) * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t t_lane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + t_lane + x * kT2Keys;
    const uint32_t t_o = tmem + t_lane + 2 * kT2Keys + x * D;
    const int r = rt * kT2Rows + x * kT2TileRows + trow;
    {  // this row of Q into shared memory, 128-byte swizzled, K-major
      const uint4* src = nullptr;
      if (r < Rb) {
        int i, h;
        row_of(a, b, hk, r, i, h);
        src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                             ((q_row0(a, b) + i) * a.Hq + h) * D);
      }
      uint4 qv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) qv[c] = src ? src[c] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int hf = c >> 3, cc = c & 7;
        uint8_t* dst = base_ptr + x * S::kQTile + hf * S::kQHalf + (trow >> 3) * 1024 +
                       (trow & 7) * 128 + ((cc ^ (trow & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = qv[c];
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }
    float m_used = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < n_it; ++j) {
      // Tile j's metadata first: the producer published it before loading K_j,
      // so this wait overlaps the wait for S_j instead of following it.
      const int st = j % kT2Meta;
      mbar_wait(&meta_bar[st], (j / kT2Meta) & 1, &abort_flag);
      const bool tile_full = meta_full[st] != 0;
      if (!mbar_wait(&s_full[x], j & 1, &abort_flag)) break;
      // lanes leave their waits at different times; the TMEM loads below are
      // warp-collective (.sync.aligned) and need the warp converged
      __syncwarp();
      tc_fence_after();
      float sv[kT2Keys];
#pragma unroll
      for (int c = 0; c < kT2Keys / 32; ++c) {
        float t[32];
        tmem_ld32(t_s + c * 32, t);
#pragma unroll
        for (int k = 0; k < 32; ++k) sv[c * 32 + k] = t[k];
      }
      tmem_wait_ld();
      const int chunk = a.chunk;
      if (!tile_full) {  // keys outside the key set: raw score -inf
#pragma unroll
        for (int k = 0; k < kT2Keys; ++k) {
          const int ci = k / chunk;
          if (k - ci * chunk >= meta[st][ci]) sv[k] = -INFINITY;
        }
      }
      // Row maximum of the raw scores (scale > 0 keeps the order): eight
      // independent three-input chains, then a short tree.
      float mx;
      {
        float m8[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) m8[g] = sv[g];
#pragma unroll
        for (int k = 8; k < kT2Keys; k += 16)
#pragma unroll
          for (int g = 0; g < 8; ++g) m8[g] = fmax3(m8[g], sv[k + g], sv[k + 8 + g]);
        mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        mx *= a.scale_log2;
      }
      if (!tile_full && x == 0) {
        // the V row of a key outside the key set may hold any bits: zero it
        // (tile A's softmax does it; PV_B(j) is issued after PV_A(j))
        // (V_j's TMA copy must have landed first; its slot is not freed before
        // PV_B(j), so its barrier cannot have moved on)
        const int vn = 2 * j + 1;
        mbar_wait(&full_bar[vn % kT2Slots], (vn / kT2Slots) & 1, &abort_flag);
        const int ci = trow / chunk;
        if (trow - ci * chunk >= meta[st][ci]) {
          uint8_t* vrow = base_ptr + (sKV0 - base) + (vn % kT2Slots) * S::kKVTile +
                          (trow >> 3) * 1024 + (trow & 7) * 128;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              *reinterpret_cast<uint4*>(vrow + hf * S::kKVHalf + (cc << 4)) =
                  make_uint4(0u, 0u, 0u, 0u);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
      }
      const float m_new = fmaxf(m_used, mx);
      // Rescale when this row's maximum grew by more than 2^8. TMEM loads and
      // stores are warp-collective, so the decision is per warp: if any row
      // needs it, every lane rescales, the others by exactly 1.
      const bool need = m_new > m_used + kT2Rescale;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;  // 0 if nothing accumulated
        if (j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= alpha;
            tmem_st32(t_o + c * 32, o);
          }
        }
        if (need) {
          l_sum *= alpha;
          m_used = m_new;
        }
      }
      const float bse = (m_used == -INFINITY) ? 0.f : m_used;
      // P = 2^(s * scale_log2 - m): one packed FMA per key pair, 2^x on the
      // MUFU (moving 3 of 8 pairs to a cubic on the FMA pipe measured slower:
      // the exponential unit is not the limit here, issue slots are). Row sums
      // in four packed chains.
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nb2 = make_float2(-bse, -bse);
      float2 lacc[4];
#pragma unroll
      for (int c = 0; c < kT2Keys / 32; ++c) {
        uint32_t pk[16];
        float2 lc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 xx = ffma2(make_float2(sv[c * 32 + 2 * k], sv[c * 32 + 2 * k + 1]), sc2, nb2);
          float2 pp;
          pp.x = fast_exp2(xx.x);
          pp.y = fast_exp2(xx.y);
          lc = fadd2(lc, pp);
          pk[k] = pack_bf16(pp.x, pp.y);
        }
        lacc[c] = lc;
        tmem_st16(t_s + c * 16, pk);  // P over the first 64 columns of S_X
      }
      {
        const float2 l01 = fadd2(lacc[0], lacc[1]), l23 = fadd2(lacc[2], lacc[3]);
        const float2 l4 = fadd2(l01, l23);
        l_sum += l4.x + l4.y;
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
    }
    // ---------------------------- epilogue (one row per thread) -------------------
    const bool have_o = n_it > 0 && mbar_wait(&o_done[x], 0, &abort_flag);
    __syncwarp();
    tc_fence_after();
    const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
    const float lse2 = l_sum > 0.f ? m_used + log2f(l_sum) : -INFINITY;
    long long row = -1;
    bool write = r < Rb;
    float wn = 1.f, wo = 0.f, Lfin = lse2 * kLn2;
    if (write && a.n_splits <= 1) {
      int i, h;
      row_of(a, b, hk, r, i, h);
      write = row_selected(a, b, h);
      row = (q_row0(a, b) + i) * a.Hq + h;
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
      if (have_o) {
        tmem_ld32(t_o + c * 32, o);
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
  // the block-wide barrier.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kT2Mma) tmem_free(tmem, kT2Cols);
}

}  // namespace fb
