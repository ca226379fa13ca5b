// lora_small_m.cuh — forward for few tokens (M <= 64): the layer is bound by
// reading W once from HBM (M d_in d_out x 2 FLOP on d_out d_in x 2 bytes,
// 2M FLOP/B, far below the ridge).
//
// Swap-AB on the tensor cores: each CTA owns a 128-row slice of W (128 output
// features) and a K range; per 64-wide K block one TMA stage brings
//   W tile   [128 x 64]   -> MMA A operand (M = 128 output features)
//   X tile   [128 x 64]   rows >= M zero-filled by TMA
//   A rows   [RP x 64]
// and the MMA warp issues
//   D  [128 features x N tokens] += W_tile * X_tile[0:N]^T     (Z^T partial)
//   DT [128 tokens   x RP]       += X_tile * A_rows^T          (T partial)
// The S CTAs that split K for the same feature slice form one thread-block
// cluster.  After the K loop each CTA parks its fp32 partials in shared
// memory; after a cluster barrier each CTA sums one S-th of the slice's
// features (and all of T) over the cluster's CTAs in rank order through
// distributed shared memory (deterministic), adds s T B^T, applies the
// activation and stores Y.  No global partials, no second launch, no atomics.
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "lora_linear.h"
#include "sm100.cuh"

namespace lora {

// Token counts up to this use the small-M path.
constexpr int64_t kSmallMMax = 64;
constexpr int kSmThreads = 192;      // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

struct SmallMParams {
  CUtensorMap tm_w;    // W [d_out x d_in], box 64 x 128
  CUtensorMap tm_x;    // X [M x d_in],     box 64 x 128
  CUtensorMap tm_a;    // A [r x d_in],     box 64 x RP
  const __nv_bfloat16* B;   // [d_out x r]
  __nv_bfloat16* Y;         // [M x d_out]
  float* T_save;            // [M x r] or null
  float* Z_save;            // [M x d_out] or null (SiLU)
  uint32_t* status;
  int M, d_in, d_out, r;
  float s;
  int act;                  // LORA_ACT_IDENTITY or LORA_ACT_SILU
  int splits;               // cluster size (K splits)
  int kb_per_split;
};

template <int kNT, int kRP>
struct SmallMCfg {
  static constexpr int kWBytes = 128 * 64 * 2;
  static constexpr int kXBytes = 128 * 64 * 2;
  static constexpr int kABytes = kRP * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes + kABytes;
  static constexpr int kStages0 = (kSmemLimitBytes - 2048) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + 2048;
  // epilogue buffers alias the ring once the K loop is done
  static constexpr int kDpBytes = 128 * kNT * 4;        // Z^T partial [128 features][kNT tokens]
  static constexpr int kTpBytes = 128 * kRP * 4;        // T partial   [128 tokens][kRP]
  static_assert(kDpBytes + 2 * kTpBytes <= kStages * kStageBytes, "epilogue buffers must fit the ring");
  static constexpr uint32_t kTmemCols = (kNT + kRP) <= 32 ? 32 : ((kNT + kRP) <= 64 ? 64 : 128);
};

template <int kNT, int kRP>
__global__ void __launch_bounds__(kSmThreads, 1) small_m_kernel(const __grid_constant__ SmallMParams p) {
  using C = SmallMCfg<kNT, kRP>;
  constexpr int S = C::kStages;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* Dp = reinterpret_cast<float*>(smem);                          // [128][kNT]
  float* Tp = reinterpret_cast<float*>(smem + C::kDpBytes);            // [128][kRP]
  float* Tf = reinterpret_cast<float*>(smem + C::kDpBytes + C::kTpBytes);  // summed T [kNT][kRP]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const int rank = static_cast<int>(cluster.block_rank());
  const int slice = blockIdx.x / p.splits;        // 128-feature slice of W
  const int nkb_all = (p.d_in + 63) / 64;
  const int kb0 = rank * p.kb_per_split;
  int kb1 = kb0 + p.kb_per_split;
  if (kb1 > nkb_all) kb1 = nkb_all;
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t tT = tbase + kNT;     // T partial columns

  if (warp == 0) {
    if (lane == 0 && nkb > 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      RingPos rp;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        uint64_t* fb = &full[rp.stage];
        mbar_arrive_expect_tx(fb, C::kStageBytes);
        const int k0 = (kb0 + i) * 64;
        tma_load_2d_hint(st, &p.tm_w, fb, k0, slice * 128, pol_stream);
        tma_load_2d_hint(st + C::kWBytes, &p.tm_x, fb, k0, 0, pol_keep);
        tma_load_2d_hint(st + C::kWBytes + C::kXBytes, &p.tm_a, fb, k0, 0, pol_keep);
        rp.next(S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdZ = idesc_bf16(128, kNT, false, false);
      constexpr uint32_t kIdT = idesc_bf16(128, kRP, false, false);
      RingPos rp;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sw = smem_u32(smem + rp.stage * C::kStageBytes);
        const uint32_t sx = sw + C::kWBytes;
        const uint32_t sa = sx + C::kXBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t dw = sdesc_sw128(sw + kk * 32, 16, 1024);
          const uint64_t dx = sdesc_sw128(sx + kk * 32, 16, 1024);
          const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
          const uint32_t acc = (i == 0 && kk == 0) ? 0u : 1u;
          mma_bf16(tbase, dw, dx, kIdZ, acc);     // Z^T partial: features x tokens
          mma_bf16(tT, dx, da, kIdT, acc);        // T partial: tokens x rank
        }
        mma_commit(&empty[rp.stage]);
        rp.next(S);
      }
      if (ok) mma_commit(acc_full);
      mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait(mma_done, 0, quiet);
    }
  } else {
    // Park this CTA's partials in shared memory (the ring is idle now).
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    bool have = false;
    if (nkb == 0) {
      have = true;
#pragma unroll
      for (int c = 0; c < kNT; ++c) Dp[lrow * kNT + c] = 0.0f;
#pragma unroll
      for (int c = 0; c < kRP; ++c) Tp[lrow * kRP + c] = 0.0f;
    } else if (mbar_wait(acc_full, 0, ctl)) {
      have = true;
      tc_fence_after();
      fence_proxy_async_smem();   // the ring was last written by TMA
      __syncwarp();
      const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < kNT; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tl + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) Dp[lrow * kNT + c0 + c] = __uint_as_float(v[c]);
      }
#pragma unroll
      for (int c0 = 0; c0 < kRP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tl + kNT + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) Tp[lrow * kRP + c0 + c] = __uint_as_float(v[c]);
      }
    }
    if (!have) {
#pragma unroll
      for (int c = 0; c < kNT; ++c) Dp[lrow * kNT + c] = 0.0f;
#pragma unroll
      for (int c = 0; c < kRP; ++c) Tp[lrow * kRP + c] = 0.0f;
    }
  }
  tc_fence_before();
  // Every CTA of the cluster has parked its partials.
  cluster.sync();

  if (warp >= 2) {
    const int et = threadIdx.x - 64;       // 0..127
    // Full T = sum over ranks of the T partials, in rank order.
    for (int i = et; i < kNT * kRP; i += 128) {
      const int m = i / kRP, c = i % kRP;
      float acc = 0.0f;
      for (int q = 0; q < p.splits; ++q) acc += cluster.map_shared_rank(Tp, q)[m * kRP + c];
      Tf[m * kRP + c] = acc;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (slice == 0 && rank == 0 && p.T_save != nullptr) {
      for (int i = et; i < p.M * p.r; i += 128) {
        const int m = i / p.r, c = i % p.r;
        p.T_save[i] = Tf[m * kRP + c];
      }
    }
    // This CTA finishes features [f0, f1) of the slice for every token.
    const int per = 128 / p.splits;
    const int f0 = rank * per;
    for (int i = et; i < per * p.M; i += 128) {
      const int m = i / per;
      const int fl = f0 + i % per;                 // feature within the slice
      const int n = slice * 128 + fl;              // output feature
      if (n >= p.d_out) continue;
      float z = 0.0f;
      for (int q = 0; q < p.splits; ++q) z += cluster.map_shared_rank(Dp, q)[fl * kNT + m];
      float lora = 0.0f;
      const __nv_bfloat16* brow = p.B + static_cast<size_t>(n) * p.r;
      for (int c = 0; c < p.r; ++c) lora += __bfloat162float(brow[c]) * Tf[m * kRP + c];
      z += p.s * lora;
      if (p.act == LORA_ACT_SILU) {
        if (p.Z_save != nullptr) p.Z_save[static_cast<size_t>(m) * p.d_out + n] = z;
        z = z / (1.0f + expf(-z));
      }
      p.Y[static_cast<size_t>(m) * p.d_out + n] = __float2bfloat16_rn(z);
    }
  }
  // Peers may still read this CTA's shared memory until everyone is done.
  cluster.sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

// Launch with S = p.splits CTAs per thread-block cluster (one cluster per
// 128-feature slice).  kNT: tokens padded to 16/32/64; kRP: r padded.
template <int kNT, int kRP>
cudaError_t launch_small_m_kernel(const SmallMParams& p, int slices, cudaStream_t st) {
  using C = SmallMCfg<kNT, kRP>;
  auto k = small_m_kernel<kNT, kRP>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(slices * p.splits), 1, 1);
  cfg.blockDim = dim3(kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}

inline cudaError_t launch_small_m(const SmallMParams& p, int nt, int rp, int slices, cudaStream_t st) {
  if (nt == 16) {
    if (rp == 16) return launch_small_m_kernel<16, 16>(p, slices, st);
    if (rp == 32) return launch_small_m_kernel<16, 32>(p, slices, st);
    return launch_small_m_kernel<16, 64>(p, slices, st);
  }
  if (nt == 32) {
    if (rp == 16) return launch_small_m_kernel<32, 16>(p, slices, st);
    if (rp == 32) return launch_small_m_kernel<32, 32>(p, slices, st);
    return launch_small_m_kernel<32, 64>(p, slices, st);
  }
  if (rp == 16) return launch_small_m_kernel<64, 16>(p, slices, st);
  if (rp == 32) return launch_small_m_kernel<64, 32>(p, slices, st);
  return launch_small_m_kernel<64, 64>(p, slices, st);
}

}  // namespace lora
