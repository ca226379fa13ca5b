// lora_gemm.cuh — persistent, warp-specialised tcgen05 kernel for the fused
// LoRA-adapted linear layer (forward) and its input gradient (backward dX).
//
// Forward  (per 128 x 256 output tile of Z = X W^T + s (X A^T) B^T):
//   K-loop over d_in: one TMA stage holds the X tile (128 x 64), the W tile
//   (256 x 64) and the A rows (r padded to RP, x 64).  For every 16-wide K step
//   the MMA warp issues  acc  += X W^T  (N = 256)  and  rank += X A^T (N = RP)
//   from the same X tile in shared memory, so X is read once for both.
//   Epilogue: T = rank (fp32) is saved, s*T is written as bf16 into shared
//   memory and one more MMA adds (s T) B^T (K = RP) into acc; then acc is read
//   out of TMEM, the activation applied and Y stored as bf16.
//   ("Liger-Kernel内核级优化：GPU利用率飙升至90%以上": y = Wx + B(Ax) computed
//   in one kernel with the activation as the last step.)
// Backward (per 128 x 256 tile of dX = dZ W + s (dZ B) A):
//   the same pipeline with W read as an MN-major operand (dX needs dZ W, W is
//   d_out x d_in row-major), the B^T rows as the rank operand (U = dZ B), and
//   A as the up-projection operand.
// SwiGLU: forward pairs a gate and an up projection in one 256-wide tile
//   (128 gate columns + 128 up columns of the same outputs); backward sums the
//   two projections' contributions over one K-loop that runs through both.
//
// Warp roles (320 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..9 = epilogue (two warps per 32-lane TMEM quadrant).
// Tensor memory: columns [0, 256) accumulator, [256, 256 + NPAIR*RP) rank.
#pragma once

#include "sm100.cuh"

namespace lora {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kGemmThreads = 320;

// kEpiGrad: backward dX with bf16 operands (dZ = dY exactly).
// kEpiGradF16: backward dX with fp16 dZ and fp16 W / B^T (activation backward:
//   dZ is fp32-valued and bf16 would round it too coarsely for dX).
enum EpiKind : int { kEpiIdentity = 0, kEpiSilu = 1, kEpiSwiglu = 2, kEpiGrad = 3, kEpiGradF16 = 4 };

struct GemmParams {
  CUtensorMap tm_a[2];    // M-side operand   fwd: X        bwd: dZ (per pair)
  CUtensorMap tm_w[2];    // main operand     fwd: W (K-major)  bwd: W (MN-major)
  CUtensorMap tm_r[2];    // rank operand     fwd: A rows   bwd: B^T rows
  CUtensorMap tm_up[2];   // up operand       fwd: B^T      bwd: A   (MN-major)
  int M;                  // rows of the output
  int N;                  // columns of the output (per pair for forward SwiGLU)
  int K;                  // reduction length (per pair)
  int r;                  // adapter rank (columns saved to rank_save)
  float s;                // LoRA scale
  __nv_bfloat16* out;     // [M x N] bf16
  float* rank_save;       // [npair][M x r] fp32 or null (rank columns computed in the K-loop)
  const float* rank_in;   // [npair][M x r] fp32: rank columns computed beforehand (kRankGlobal)
  float* z_save;          // [npair][M x N] fp32 or null (forward SiLU / SwiGLU)
  uint32_t* status;       // device status word or null
  int m_tiles, n_tiles, num_tiles, group_m;
};

// kRankGlobal == false: the rank columns T = X A^T (U = dZ B) ride the K-loop as
//   extra MMA columns (X read from HBM once; costs RP/256 extra tensor work).
// kRankGlobal == true: T (U) was computed by a rank pass; the epilogue loads it.
template <bool kBwd, int kRP, int kNPair, int kEpi, bool kRankGlobal>
struct GemmCfg {
  static constexpr bool kSwigluFwd = (!kBwd) && (kEpi == kEpiSwiglu);
  static constexpr int kOutCols = kSwigluFwd ? 128 : 256;           // output columns per tile
  static constexpr int kKPairs = kBwd ? kNPair : 1;                 // pairs walked along K
  static constexpr int kRankRows = kRankGlobal ? 0 : (kSwigluFwd ? 2 * kRP : kRP);  // rank rows per stage
  static constexpr int kUpCols = kSwigluFwd ? 128 : 256;            // N of one up-projection MMA
  static constexpr int kABytes = kBM * kBK * 2;                     // 16 KB
  static constexpr int kWBytes = kBN * kBK * 2;                     // 32 KB
  static constexpr int kRBytes = kRankRows * kBK * 2;
  static constexpr int kStageBytes = kABytes + kWBytes + kRBytes;   // multiple of 1 KB
  static constexpr int kUpTx = (kUpCols / 64) * kRP * 128;
  static constexpr int kBarBytes = 1024;
  static constexpr int kStages0 = (kSmemLimitBytes - 1024 - kBarBytes) / kStageBytes;
  static constexpr int kStages = kStages0 > 6 ? 6 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
  static constexpr int kRankCols = kRankGlobal ? 0 : kNPair * kRP;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1 KB alignment");
  static_assert(kRP % 16 == 0 && kRP <= 64, "rank padding");
  static_assert(kStages >= 2, "not enough shared memory");
  static_assert(256 + kRankCols <= 512, "tensor memory budget");
  static_assert(kUpTx <= kWBytes, "up operand must fit the W area of a stage");
};

__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& mt, int& nt) {
  const int per_group = p.group_m * p.n_tiles;
  const int g = t / per_group;
  const int first_m = g * p.group_m;
  const int rem = p.m_tiles - first_m;
  const int gm = rem < p.group_m ? rem : p.group_m;
  const int idx = t - g * per_group;
  mt = first_m + idx % gm;
  nt = idx / gm;
}

template <bool kBwd, int kRP, int kNPair, int kEpi, bool kRankGlobal>
__global__ void __launch_bounds__(kGemmThreads, 1) lora_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg<kBwd, kRP, kNPair, kEpi, kRankGlobal>;
  constexpr bool kRankLoop = (kRP > 0) && !kRankGlobal;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* full = bars;                  // [S]
  uint64_t* empty = bars + S;             // [S]
  uint64_t* acc_full = bars + 2 * S;      // rank columns ready (K-loop done)
  uint64_t* acc_final = acc_full + 1;     // accumulator complete (up-projection done)
  uint64_t* acc_empty = acc_full + 2;     // epilogue drained TMEM
  uint64_t* rank_ready = acc_full + 3;    // [2] s*rank written to shared memory
  uint64_t* mma_done = acc_full + 5;      // teardown: all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 6);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_final, 1);
    mbar_init(acc_empty, 256);
    mbar_init(&rank_ready[0], 128);
    mbar_init(&rank_ready[1], 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < (C::kSwigluFwd ? 1 : kNPair); ++j) tma_prefetch_desc(&p.tm_a[j]);
    for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_w[j]);
    if (kRankLoop) for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_r[j]);
    if (kRP > 0) for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_up[j]);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int nkb = (p.K + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      RingPos rp;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, p, mt, nt);
        const int m0 = mt * kBM, n0 = nt * C::kOutCols;
        for (int j = 0; j < C::kKPairs && ok; ++j) {
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) { ok = false; break; }
            uint8_t* sa = smem + rp.stage * C::kStageBytes;
            uint8_t* sw = sa + C::kABytes;
            uint8_t* sr = sw + C::kWBytes;
            uint64_t* fb = &full[rp.stage];
            mbar_arrive_expect_tx(fb, C::kStageBytes);
            const int k0 = kb * kBK;
            tma_load_2d_hint(sa, &p.tm_a[j], fb, k0, m0, pol_stream);
            if constexpr (!kBwd) {
              if constexpr (C::kSwigluFwd) {
                tma_load_2d_hint(sw, &p.tm_w[0], fb, k0, n0, pol_keep);
                tma_load_2d_hint(sw + C::kWBytes / 2, &p.tm_w[1], fb, k0, n0, pol_keep);
              } else {
                tma_load_2d_hint(sw, &p.tm_w[0], fb, k0, n0, pol_keep);
              }
              if constexpr (kRankLoop) {
                tma_load_2d_hint(sr, &p.tm_r[0], fb, k0, 0, pol_keep);
                if constexpr (C::kSwigluFwd) tma_load_2d_hint(sr + kRP * 128, &p.tm_r[1], fb, k0, 0, pol_keep);
              }
            } else {
#pragma unroll
              for (int b = 0; b < 4; ++b) tma_load_2d_hint(sw + b * 8192, &p.tm_w[j], fb, n0 + 64 * b, k0, pol_keep);
              if constexpr (kRankLoop) tma_load_2d_hint(sr, &p.tm_r[j], fb, k0, 0, pol_keep);
            }
            ++issued;
            rp.next(S);
          }
        }
        if constexpr (kRP > 0) {
          for (int j = 0; j < kNPair && ok; ++j) {
            if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) { ok = false; break; }
            uint8_t* sw = smem + rp.stage * C::kStageBytes + C::kABytes;
            uint64_t* fb = &full[rp.stage];
            mbar_arrive_expect_tx(fb, C::kUpTx);
            const int nup = C::kSwigluFwd ? n0 : n0;
#pragma unroll
            for (int b = 0; b < C::kUpCols / 64; ++b)
              tma_load_2d_hint(sw + b * (kRP * 128), &p.tm_up[j], fb, nup + 64 * b, 0, pol_keep);
            ++issued;
            rp.next(S);
          }
        }
      }
      if (!ok) {
        // Let copies already issued land before the CTA exits.
        RingPos q = rp;
        AbortCtl quiet{nullptr, nullptr};
        volatile uint32_t zero = 0u;
        quiet.flag = &zero;
        for (uint32_t i = 0; i < (issued < (uint32_t)S ? issued : (uint32_t)S); ++i) {
          if (q.stage == 0) { q.stage = S - 1; q.phase ^= 1u; } else { --q.stage; }
          mbar_wait(&full[q.stage], q.phase, quiet);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool kF16 = (kEpi == kEpiGradF16);
      constexpr uint32_t kIdMain = idesc_mma(128, 256, false, kBwd, kF16);
      constexpr uint32_t kIdRank =
          idesc_mma(128, C::kSwigluFwd ? 2 * (kRP > 0 ? kRP : 8) : (kRP > 0 ? kRP : 16), false, false, kF16);
      constexpr uint32_t kIdUp = idesc_bf16(128, C::kUpCols, false, true);
      RingPos rp;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, ctl)) break;
        tc_fence_after();
        bool ok = true;
        uint32_t first_main = 1;
        for (int j = 0; j < C::kKPairs && ok; ++j) {
          const uint32_t trank = tbase + 256 + (kBwd ? j * kRP : 0);
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
            const uint32_t sw = sa + C::kABytes;
            const uint32_t sr = sw + C::kWBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t dw = kBwd ? sdesc_sw128(sw + kk * 2048, 8192, 1024) : sdesc_sw128(sw + kk * 32, 16, 1024);
              mma_bf16(tbase, da, dw, kIdMain, (first_main && kk == 0) ? 0u : 1u);
              if constexpr (kRankLoop) {
                const uint64_t dr = sdesc_sw128(sr + kk * 32, 16, 1024);
                mma_bf16(trank, da, dr, kIdRank, (kb == 0 && kk == 0) ? 0u : 1u);
              }
            }
            first_main = 0;
            mma_commit(&empty[rp.stage]);
            rp.next(S);
          }
        }
        if (!ok) break;
        if constexpr (kRP > 0) {
          // K-loop done: the epilogue may now use this tile's up-projection
          // slots (waiting on them earlier could alias an older phase).
          mma_commit(acc_full);
          for (int j = 0; j < kNPair && ok; ++j) {
            if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
            if (!mbar_wait(&rank_ready[j], acc_phase, ctl)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
            const uint32_t su = sa + C::kABytes;
            const uint32_t dcol = C::kSwigluFwd ? static_cast<uint32_t>(j * 128) : 0u;
#pragma unroll
            for (int kk = 0; kk < kRP / 16; ++kk) {
              const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t du = sdesc_sw128(su + kk * 2048, kRP * 128, 1024);
              mma_bf16(tbase + dcol, da, du, kIdUp, 1u);
            }
            mma_commit(&empty[rp.stage]);
            rp.next(S);
          }
          if (!ok) break;
        }
        mma_commit(acc_final);
        acc_phase ^= 1u;
      }
      // Teardown: every MMA issued by this thread retires before TMEM is freed.
      mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait(mma_done, 0, quiet);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..7
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int h = ew >> 2;                   // column half
    const int row_in_tile = q * 32 + lane;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(q * 32) << 16);
    RingPos rp;
    uint32_t acc_phase = 0;
    const int nkb_total = nkb * C::kKPairs;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, p, mt, nt);
      const int row = mt * kBM + row_in_tile;
      const bool row_ok = row < p.M;
      // Skip the ring positions of the K-loop.
      for (int i = 0; i < nkb_total; ++i) rp.next(S);
      if constexpr (kRP > 0) {
        float rk[kRP];
        if constexpr (!kRankLoop) {
          // Rank values computed by the rank pass: fetch them while the K-loop runs.
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
        // The up-projection slots of this tile are only safe to wait on once the
        // K-loop is done: before that a slot's barrier may be two phases behind,
        // where a parity wait would return early.
        if (!mbar_wait(acc_full, acc_phase, ctl)) break;
        tc_fence_after();
        bool ok = true;
        RingPos up = rp;
        for (int j = 0; j < kNPair; ++j) {
          if (j == h) {
            if constexpr (kRankLoop) {
              __syncwarp();   // tcgen05.ld is .sync.aligned: converge the warp first
#pragma unroll
              for (int c0 = 0; c0 < kRP; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tlane + 256 + j * kRP + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) rk[c0 + c] = __uint_as_float(v[c]);
              }
            }
            if (kRankLoop && p.rank_save != nullptr && nt == 0 && row_ok) {
              float* dst = p.rank_save + (static_cast<size_t>(j) * p.M + row) * p.r;
#pragma unroll
              for (int c = 0; c < kRP; c += 4)
                if (c < p.r) *reinterpret_cast<float4*>(dst + c) = make_float4(rk[c], rk[c + 1], rk[c + 2], rk[c + 3]);
            }
            if (!mbar_wait(&full[up.stage], up.phase, ctl)) { ok = false; }
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
              mbar_arrive(&rank_ready[j]);
            }
          }
          up.next(S);
        }
        if (!ok) break;
        rp = up;
      }
      if (!mbar_wait(acc_final, acc_phase, ctl)) break;
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
      mbar_arrive(acc_empty);
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

}  // namespace lora
