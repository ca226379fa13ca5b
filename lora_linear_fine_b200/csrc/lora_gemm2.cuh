// lora_gemm2.cuh — the LoRA-linear GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation and warp roles as lora_gemm_kernel (lora_gemm.cuh), but a
// thread-block cluster of two CTAs on two SMs computes one 256 x 256 tile:
//   CTA c (c = 0, 1) holds rows [128c, 128c + 128) of the M-side operand (X or
//   dZ) and half of the N-side operand (W rows / columns [128c, 128c + 128),
//   or for the SwiGLU forward the gate (c = 0) or up (c = 1) weight rows);
//   CTA 0 (the leader) issues tcgen05.mma.cta_group::2 with M = 256, N = 256;
//   each CTA's tensor memory receives its own 128 accumulator rows.
// Per 64-wide K block each CTA moves 32 KB through shared memory instead of
// 48 KB for the same tensor work per SM, so the TMA ring is deeper and the
// L2 -> SM stream two thirds as large.
//
// Synchronisation across the pair:
//   * each CTA loads its own halves; the transactions complete on the leader's
//     `full` barrier (the leader announces both halves' bytes);
//   * the leader's commits arrive on `empty`, `acc_full`, `acc_final` of both
//     CTAs (multicast commit);
//   * both CTAs' epilogue threads arrive on the leader's `acc_empty` and
//     `rank_ready` barriers through their cluster addresses;
//   * the up-projection operand s*T (or s*U) is written by each CTA's epilogue
//     into its own shared memory; the leader's MMA reads both halves.
#pragma once

#include "lora_gemm.cuh"

namespace lora {

template <bool kBwd, int kRP, int kNPair, int kEpi, bool kRankGlobal>
struct Gemm2Cfg {
  static constexpr bool kSwigluFwd = (!kBwd) && (kEpi == kEpiSwiglu);
  static constexpr int kOutCols = kSwigluFwd ? 128 : 256;        // output columns per pair tile
  static constexpr int kKPairs = kBwd ? kNPair : 1;
  static constexpr int kRankRowsHalf = kRankGlobal ? 0 : kRP / 2;  // rank operand rows per CTA
  static constexpr int kUpCols = kSwigluFwd ? 128 : 256;         // N of one up-projection MMA (pair)
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBBytes = 128 * 64 * 2;
  static constexpr int kRBytes = kRankRowsHalf * 128;
  static constexpr int kStageBytes = kABytes + kBBytes + kRBytes;
  static constexpr int kUpBoxes = kUpCols / 2 / 64;               // 64-wide boxes per CTA
  static constexpr int kUpTxHalf = kUpBoxes * kRP * 128;
  static constexpr int kStages0 = (kSmemLimitBytes - 2048) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + 2048;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kRankGlobal || (kRP == 16 && !kSwigluFwd && kNPair == 1), "in-loop rank columns: RP = 16 only");
  static_assert(kUpTxHalf <= kBBytes, "up operand half must fit the B area");
  static_assert(kStages >= 3, "ring too shallow");
};

template <bool kBwd, int kRP, int kNPair, int kEpi, bool kRankGlobal>
__global__ void __launch_bounds__(kGemmThreads, 1) lora_gemm2_kernel(const __grid_constant__ GemmParams p) {
  using C = Gemm2Cfg<kBwd, kRP, kNPair, kEpi, kRankGlobal>;
  constexpr int S = C::kStages;
  constexpr bool kRankLoop = (kRP > 0) && !kRankGlobal;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* full = bars;                  // [S]  (the leader's are used)
  uint64_t* empty = bars + S;             // [S]  (both CTAs')
  uint64_t* acc_full = bars + 2 * S;      // K-loop done (both CTAs')
  uint64_t* acc_final = acc_full + 1;     // accumulator complete (both CTAs')
  uint64_t* acc_empty = acc_full + 2;     // tensor memory drained (leader's, 2 x 256 arrivals)
  uint64_t* rank_ready = acc_full + 3;    // [2] s*rank written (leader's, 2 x 128 arrivals)
  uint64_t* mma_done = acc_full + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 6);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const bool leader = crank == 0;
  const int cluster_id = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  AbortCtl ctl{abort_flag, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_final, 1);
    mbar_init(acc_empty, 512);
    mbar_init(&rank_ready[0], 256);
    mbar_init(&rank_ready[1], 256);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < (C::kSwigluFwd ? 1 : kNPair); ++j) tma_prefetch_desc(&p.tm_a[j]);
    for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_w[j]);
    if (kRankLoop) tma_prefetch_desc(&p.tm_r[0]);
    if (kRP > 0) for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_up[j]);
  }
  if (warp == 1) { tmem_alloc_pair(tmem_slot, C::kTmemCols); tmem_relinquish_pair(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int nkb = (p.K + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      RingPos rp;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = cluster_id; t < p.num_tiles && ok; t += nclusters) {
        int mt, nt;
        tile_coords(t, p, mt, nt);
        const int m0 = mt * 256 + 128 * static_cast<int>(crank);
        const int n0 = nt * C::kOutCols;
        for (int j = 0; j < C::kKPairs && ok; ++j) {
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait_cluster(&empty[rp.stage], rp.phase ^ 1u, ctl)) { ok = false; break; }
            uint8_t* sa = smem + rp.stage * C::kStageBytes;
            uint8_t* sb = sa + C::kABytes;
            uint8_t* sr = sb + C::kBBytes;
            if (leader) mbar_arrive_expect_tx(&full[rp.stage], 2 * C::kStageBytes);
            const uint32_t fb = mapa_shared(smem_u32(&full[rp.stage]), 0);
            const int k0 = kb * kBK;
            tma_load_2d_pair(sa, &p.tm_a[j], fb, k0, m0, pol_stream);
            if constexpr (!kBwd) {
              if constexpr (C::kSwigluFwd) tma_load_2d_pair(sb, &p.tm_w[crank], fb, k0, n0, pol_keep);
              else tma_load_2d_pair(sb, &p.tm_w[0], fb, k0, n0 + 128 * static_cast<int>(crank), pol_keep);
            } else {
#pragma unroll
              for (int b = 0; b < 2; ++b)
                tma_load_2d_pair(sb + b * 8192, &p.tm_w[j], fb, n0 + 128 * static_cast<int>(crank) + 64 * b, k0,
                                 pol_keep);
            }
            if constexpr (kRankLoop)
              tma_load_2d_pair(sr, &p.tm_r[0], fb, k0, C::kRankRowsHalf * static_cast<int>(crank), pol_keep);
            ++issued;
            rp.next(S);
          }
        }
        if constexpr (kRP > 0) {
          for (int j = 0; j < kNPair && ok; ++j) {
            if (!mbar_wait_cluster(&empty[rp.stage], rp.phase ^ 1u, ctl)) { ok = false; break; }
            uint8_t* sb = smem + rp.stage * C::kStageBytes + C::kABytes;
            if (leader) mbar_arrive_expect_tx(&full[rp.stage], 2 * C::kUpTxHalf);
            const uint32_t fb = mapa_shared(smem_u32(&full[rp.stage]), 0);
            const int nstart = n0 + (C::kUpCols / 2) * static_cast<int>(crank);
#pragma unroll
            for (int b = 0; b < C::kUpBoxes; ++b)
              tma_load_2d_pair(sb + b * (kRP * 128), &p.tm_up[j], fb, nstart + 64 * b, 0, pol_keep);
            ++issued;
            rp.next(S);
          }
        }
      }
      if (!ok && leader) {
        // The leader's full barriers count both CTAs' copies: let them land.
        RingPos q = rp;
        volatile uint32_t zero = 0u;
        AbortCtl quiet{&zero, nullptr};
        for (uint32_t i = 0; i < (issued < (uint32_t)S ? issued : (uint32_t)S); ++i) {
          if (q.stage == 0) { q.stage = S - 1; q.phase ^= 1u; } else { --q.stage; }
          mbar_wait_cluster(&full[q.stage], q.phase, quiet);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr bool kF16 = (kEpi == kEpiGradF16);
      constexpr uint32_t kIdMain = idesc_mma(256, 256, false, kBwd, kF16);
      constexpr uint32_t kIdRank = idesc_mma(256, kRP > 0 ? kRP : 16, false, false, kF16);
      constexpr uint32_t kIdUp = idesc_bf16(256, C::kUpCols, false, true);
      constexpr uint16_t kBoth = 0x3;
      RingPos rp;
      uint32_t acc_phase = 0;
      for (int t = cluster_id; t < p.num_tiles; t += nclusters) {
        if (!mbar_wait_cluster(acc_empty, acc_phase ^ 1u, ctl)) break;
        tc_fence_after();
        bool ok = true;
        uint32_t first_main = 1;
        for (int j = 0; j < C::kKPairs && ok; ++j) {
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait_cluster(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
            const uint32_t sb = sa + C::kABytes;
            const uint32_t sr = sb + C::kBBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t db = kBwd ? sdesc_sw128(sb + kk * 2048, 8192, 1024) : sdesc_sw128(sb + kk * 32, 16, 1024);
              mma_bf16_pair(tbase, da, db, kIdMain, (first_main && kk == 0) ? 0u : 1u);
              if constexpr (kRankLoop) {
                const uint64_t dr = sdesc_sw128(sr + kk * 32, 16, 1024);
                mma_bf16_pair(tbase + 256, da, dr, kIdRank, (kb == 0 && kk == 0) ? 0u : 1u);
              }
            }
            first_main = 0;
            mma_commit_pair(&empty[rp.stage], kBoth);
            rp.next(S);
          }
        }
        if (!ok) break;
        if constexpr (kRP > 0) {
          mma_commit_pair(acc_full, kBoth);
          for (int j = 0; j < kNPair && ok; ++j) {
            if (!mbar_wait_cluster(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
            if (!mbar_wait_cluster(&rank_ready[j], acc_phase, ctl)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
            const uint32_t su = sa + C::kABytes;
            const uint32_t dcol = C::kSwigluFwd ? static_cast<uint32_t>(j * 128) : 0u;
#pragma unroll
            for (int kk = 0; kk < kRP / 16; ++kk) {
              const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t du = sdesc_sw128(su + kk * 2048, kRP * 128, 1024);
              mma_bf16_pair(tbase + dcol, da, du, kIdUp, 1u);
            }
            mma_commit_pair(&empty[rp.stage], kBoth);
            rp.next(S);
          }
          if (!ok) break;
        }
        mma_commit_pair(acc_final, kBoth);
        acc_phase ^= 1u;
      }
      mma_commit_pair(mma_done, 0x1);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait_cluster(mma_done, 0, quiet);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;
    const int q = warp & 3;
    const int h = ew >> 2;
    const int row_in_tile = q * 32 + lane;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    RingPos rp;
    uint32_t acc_phase = 0;
    const int nkb_total = nkb * C::kKPairs;
    for (int t = cluster_id; t < p.num_tiles; t += nclusters) {
      int mt, nt;
      tile_coords(t, p, mt, nt);
      const int row = mt * 256 + 128 * static_cast<int>(crank) + row_in_tile;
      const bool row_ok = row < p.M;
      for (int i = 0; i < nkb_total; ++i) rp.next(S);
      if constexpr (kRP > 0) {
        float rk[kRP];
        if constexpr (!kRankLoop) {
          if (h < kNPair) {
            const float* src = p.rank_in + (static_cast<size_t>(h) * p.M + row) * p.r;
#pragma unroll
            for (int c = 0; c < kRP; c += 4) {
              float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
              if (row_ok && c < p.r) v4 = *reinterpret_cast<const float4*>(src + c);
              rk[c] = v4.x; rk[c + 1] = v4.y; rk[c + 2] = v4.z; rk[c + 3] = v4.w;
            }
          }
        }
        // Wait for the K-loop first: the up slot's barriers are then at most one phase behind.
        if (!mbar_wait_cluster(acc_full, acc_phase, ctl)) break;
        tc_fence_after();
        bool ok = true;
        RingPos up = rp;
        for (int j = 0; j < kNPair; ++j) {
          if (j == h) {
            if constexpr (kRankLoop) {
              __syncwarp();
#pragma unroll
              for (int c0 = 0; c0 < kRP; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tlane + 256 + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) rk[c0 + c] = __uint_as_float(v[c]);
              }
              if (p.rank_save != nullptr && nt == 0 && row_ok) {
                float* dst = p.rank_save + static_cast<size_t>(row) * p.r;
#pragma unroll
                for (int c = 0; c < kRP; c += 4)
                  if (c < p.r) *reinterpret_cast<float4*>(dst + c) = make_float4(rk[c], rk[c + 1], rk[c + 2], rk[c + 3]);
              }
            }
            // The slot's previous use has been consumed (this CTA's copy of `empty`).
            if (!mbar_wait_cluster(&empty[up.stage], up.phase ^ 1u, ctl)) { ok = false; }
            if (ok) {
              uint8_t* sa = smem + up.stage * C::kStageBytes;
#pragma unroll
              for (int c = 0; c < kRP; c += 8) {
                uint4 pk;
                pk.x = pack_bf16x2(p.s * rk[c + 0], p.s * rk[c + 1]);
                pk.y = pack_bf16x2(p.s * rk[c + 2], p.s * rk[c + 3]);
                pk.z = pack_bf16x2(p.s * rk[c + 4], p.s * rk[c + 5]);
                pk.w = pack_bf16x2(p.s * rk[c + 6], p.s * rk[c + 7]);
                *reinterpret_cast<uint4*>(sa + sw128_offset(row_in_tile, c)) = pk;
              }
              fence_proxy_async_smem();
              mbar_arrive_cluster(mapa_shared(smem_u32(&rank_ready[j]), 0));
            }
          }
          up.next(S);
        }
        if (!ok) break;
        rp = up;
      }
      if (!mbar_wait_cluster(acc_final, acc_phase, ctl)) break;
      tc_fence_after();
      __syncwarp();
      uint32_t v[128];
      if constexpr (C::kSwigluFwd) {
        tmem_ld32(tlane + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tlane + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld32(tlane + 128 + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
        tmem_ld32(tlane + 128 + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tlane + h * 128 + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_cluster(acc_empty_leader);
      acc_phase ^= 1u;
      if (!row_ok) continue;

      if constexpr (C::kSwigluFwd) {
        const int col0 = nt * 128 + h * 64;
        const size_t base = static_cast<size_t>(row) * p.N + col0;
        if (p.z_save != nullptr) {
          float* zg = p.z_save + base;
          float* zu = p.z_save + static_cast<size_t>(p.M) * p.N + base;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            if (col0 + c < p.N) {
              *reinterpret_cast<float4*>(zg + c) = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                               __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
              *reinterpret_cast<float4*>(zu + c) =
                  make_float4(__uint_as_float(v[64 + c]), __uint_as_float(v[65 + c]), __uint_as_float(v[66 + c]),
                              __uint_as_float(v[67 + c]));
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          float hv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float g = __uint_as_float(v[c + e]);
            const float u = __uint_as_float(v[64 + c + e]);
            hv[e] = g / (1.0f + expf(-g)) * u;
          }
          if (col0 + c < p.N) {
            uint4 pk;
            pk.x = pack_bf16x2(hv[0], hv[1]);
            pk.y = pack_bf16x2(hv[2], hv[3]);
            pk.z = pack_bf16x2(hv[4], hv[5]);
            pk.w = pack_bf16x2(hv[6], hv[7]);
            *reinterpret_cast<uint4*>(p.out + base + c) = pk;
          }
        }
      } else {
        const int col0 = nt * 256 + h * 128;
        const size_t base = static_cast<size_t>(row) * p.N + col0;
        if constexpr (kEpi == kEpiSilu) {
          if (p.z_save != nullptr) {
#pragma unroll
            for (int c = 0; c < 128; c += 4)
              if (col0 + c < p.N)
                *reinterpret_cast<float4*>(p.z_save + base + c) =
                    make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2]),
                                __uint_as_float(v[c + 3]));
          }
        }
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          float yv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float z = __uint_as_float(v[c + e]);
            yv[e] = (kEpi == kEpiSilu) ? z / (1.0f + expf(-z)) : z;
          }
          if (col0 + c < p.N) {
            uint4 pk;
            pk.x = pack_bf16x2(yv[0], yv[1]);
            pk.y = pack_bf16x2(yv[2], yv[3]);
            pk.z = pack_bf16x2(yv[4], yv[5]);
            pk.w = pack_bf16x2(yv[6], yv[7]);
            *reinterpret_cast<uint4*>(p.out + base + c) = pk;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its peer may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, C::kTmemCols);
  }
}

}  // namespace lora
