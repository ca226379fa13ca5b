// lora_small_m.cuh — forward for few tokens (M <= 64).  With so few tokens the
// layer is bound by reading W once from HBM (2 M d_in d_out FLOP on about
// 2 d_in d_out bytes), so the kernel is laid out for bandwidth and for a
// short tail after the stream.
//
// One thread-block cluster of S CTAs per 128-row slice of W (S = 1..16, one
// CTA per SM); the CTAs of a cluster split the K dimension.  One TMA stage
// brings kKPS 64-wide K blocks (two for a bf16 weight: 32 KB of W per stage
// and per barrier round trip, which streams measurably faster than 16 KB
// stages), each as
//   X tile [kNT tokens x 64], rows >= M zero
//   A tile [a_rows x 64], a_rows = r rounded up to 16, rows >= r zero
//   W tile [128 rows x 64]
// and two MMAs per 16-wide K step:
//   Z^T partial  D_Z [128 x kNT]    += W X^T   (swap-AB: the weight rows are
//                                              the M side, the tokens N)
//   T partial    D_T [128 x a_rows] += X A^T   (M = a 128-row window from the
//                                              X slot's start, which runs on
//                                              into the A and W slots of the
//                                              same block: rows >= kNT of D_T
//                                              are garbage and never read)
// Every cluster covers all of K, so each computes the full T for itself: no
// CTA outside the cluster is ever needed.  After the K loop each CTA parks its
// fp32 partials in its own shared memory; after a cluster barrier each CTA
// sums the cluster's T partials and its share of the slice's Z partials in
// rank order through distributed shared memory (deterministic, no global
// partials, no atomics), adds s T B^T, applies the activation and stores Y.
#pragma once

#include <cuda_runtime.h>

#include "lora_linear.h"
#include "lora_w4.cuh"
#include "sm100.cuh"

namespace lora {

constexpr int64_t kSmallMMax = 64;
constexpr int kSmThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kSmMaxCluster = 16;

struct SmallMParams {
  CUtensorMap tm_w;          // W [d_out x d_in], box 64 x 128; 4-bit weight: Wq [d_out x d_in/2] bytes, box 32 x 128
  CUtensorMap tm_ws;         // 4-bit weight only: scales [d_in/64 x d_out] bf16, box 128 x kKPS
  const uint8_t* Wt;         // 4-bit weight: the codes in the tiled layout (lora_w4.cuh), or null (tm_w)
  CUtensorMap tm_a;          // A [r x d_in],     box 64 x a_rows (rows >= r zero-filled)
  CUtensorMap tm_x;          // X [M x d_in],     box 64 x kNT (rows >= M zero-filled)
  // The same operands as 3D views [K blocks][rows][64] (d_in a multiple of
  // 64): box 64 x rows x kKPS, one TMA load per operand and stage
  CUtensorMap tm_x3, tm_a3, tm_w3;   // tm_a3: box kAR rows; tm_w3: bf16 weight only
  int load3d;                // 1: the 3D views are used; 0: one 2D box per K block
  const __nv_bfloat16* B;    // [d_out x r]
  __nv_bfloat16* Y;          // [M x d_out]
  float* T_save;             // [M x r] or null
  float* Z_save;             // [M x d_out] or null (SiLU)
  uint32_t* status;
  int M, d_in, d_out, r;
  float s;
  int act;
  int splits;                // CTAs per cluster (K splits)
  int kb_per;                // 64-wide K blocks per CTA
  int a_rows;                // rows of A loaded per K block: r rounded up to 16
  unsigned long long* trace; // null, or [grid][kSmTraceStride] globaltimer stamps (debugging)
};

// Trace points of one CTA (LORA_LINEAR_DEBUG=2 prints them per launch).
enum SmTrace : int {
  kTrEntry = 0, kTrFirstIssue, kTrFirstData, kTrLastMma, kTrPublished, kTrSynced, kTrTSummed, kTrCombined, kTrExit,
  kTrDqWait, kTrDqWork,   // 4-bit weight: total ns the expanding warps waited for data / spent expanding
  kSmTracePoints
};
// Per-stage stamps after the points above: when the producer issued stage i
// and when the MMA warp saw it full (the first kSmTraceStages stages).
constexpr int kSmTraceStages = 16;
constexpr int kSmTraceStride = kSmTracePoints + 2 * kSmTraceStages;

__device__ __forceinline__ unsigned long long sm_clock_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t) : : "memory");
  return t;
}

__device__ __forceinline__ void sm_trace(const SmallMParams& p, int point) {
  if (p.trace != nullptr) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t) : : "memory");
    p.trace[static_cast<size_t>(blockIdx.x) * kSmTraceStride + point] = t;
  }
}

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

// Sum of the float4 at shared offset `saddr` over the cluster's first
// `splits` CTAs, in rank order.  All loads are issued before the first add.
__device__ __forceinline__ float4 cluster_sum4(uint32_t saddr, int splits) {
  float4 v[kSmMaxCluster];
#pragma unroll
  for (int qq = 0; qq < kSmMaxCluster; ++qq)
    if (qq < splits) v[qq] = ld_dsmem_f32x4(mapa_shared(saddr, static_cast<uint32_t>(qq)));
  float4 t = v[0];
#pragma unroll
  for (int qq = 1; qq < kSmMaxCluster; ++qq)
    if (qq < splits) { t.x += v[qq].x; t.y += v[qq].y; t.z += v[qq].z; t.w += v[qq].w; }
  return t;
}

// 16 fp32 columns of this warp's TMEM lanes.
__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, float (&out)[16]) {
  uint32_t v[16];
  tmem_ld16(taddr, v);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 16; ++c) out[c] = __uint_as_float(v[c]);
}

// 64-wide K blocks per pipeline stage.  Each operand of a stage arrives in
// one TMA operation (a 3D box over consecutive K blocks), and the SM issues
// TMA operations at a roughly fixed cost each, whatever their size: so the
// 4-bit kernel, whose per-block tiles are small, takes four blocks a stage
// when its X and A tiles are small enough, the others two.
constexpr int small_m_kps(int nt, bool w4, int ar) { return w4 ? ((nt + ar) * 128 <= 4096 ? 4 : 2) : 2; }

template <int kNT, bool kW4, int kAR>
struct SmallMCfg {
  static constexpr int kKPS = small_m_kps(kNT, kW4, kAR);
  // stage = [X tiles | A tiles | W tiles (bf16) or code tiles + scale rows
  // (4-bit)], kKPS of each, every tile a SWIZZLE_128B image of its 64-wide K
  // block; the 4-bit kernel expands its codes into a short ring of W tiles
  // of its own (kWBufs), so that the small code stages can all be in flight
  static constexpr int kXBox = kNT * 64 * 2;            // X tile: kNT rows x 64
  static constexpr int kABox = kAR * 64 * 2;            // A slot: kAR >= a_rows rows x 64
  static constexpr int kWBox = 128 * 64 * 2;            // W tile: 128 rows x 64
  static constexpr int kQBox = kW4 ? 128 * 32 : 0;      // 4-bit weight: packed codes, 128 rows x 32 bytes
  static constexpr int kSBox = kW4 ? 128 * 2 : 0;       // 4-bit weight: the 128 rows' scales of one K block
  static constexpr int kXOff = 0;
  static constexpr int kAOff = kKPS * kXBox;
  static constexpr int kWOff = kAOff + kKPS * kABox;    // bf16
  static constexpr int kQOff = kWOff;                   // 4-bit
  static constexpr int kSOff = kQOff + kKPS * kQBox;    // 4-bit
  static constexpr int kStageBytes = kW4 ? (kSOff + kKPS * kSBox + 1023) / 1024 * 1024 : kWOff + kKPS * kWBox;
  // expanded W tiles (4-bit): a tile is free again only when the MMAs of the
  // block that used it have retired, so the ring must cover that latency
  // (three tiles measured short at four blocks a stage: the expanding warps
  // waited as long as they worked)
  static constexpr int kWBufs = kW4 ? (kKPS == 4 ? 6 : 3) : 0;
  static constexpr int kWRingBytes = kWBufs * kWBox;
  static constexpr int kLd = kNT + 4;                   // parked row stride (floats): 16-byte rows, conflict-free float4 stores
  static constexpr int kBsBytes = 128 * 66 * 2;         // B rows of this CTA's features, bf16, stride r + 2
  static constexpr int kTailBytes = kBsBytes + 1024 + 1024;   // B rows, barriers, alignment slack
  static constexpr int kStages0 = (kSmemLimitBytes - kTailBytes - kWRingBytes) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kWRingBytes + kTailBytes;
  static constexpr uint32_t kTmemCols = 128;            // D_Z: kNT columns, then D_T: kAR columns
  // after the K loop the ring holds: Dp [128][kLd], Tp [128][kLd], Tf [64][kNT]
  static constexpr int kParkBytes = 2 * 128 * kLd * 4 + kNT * 64 * 4;
  static_assert(kXBox % 1024 == 0 && kABox % 1024 == 0 && kWBox % 1024 == 0 && kStageBytes % 1024 == 0, "swizzle atoms");
  static_assert(kNT + kAR <= static_cast<int>(kTmemCols), "tensor memory");
  // The T product reads a 128-row window (16 KB) from an X tile; only its
  // first kNT rows are used.  From the last stage's last X tile it stays
  // inside the ring plus what follows it (the W tiles or the B rows).
  static_assert((kKPS - 1) * kXBox + 128 * 128 <= kStageBytes + kWRingBytes + kBsBytes, "T window");
  static_assert(kStages >= 3, "ring too shallow");
  static_assert(kParkBytes <= kStages * kStageBytes, "parked partials must fit the ring");
};

// kW4: the base weight arrives as 4-bit codes with one bf16 scale per row and
// 64 input features; the epilogue warps, idle during the K loop, turn each
// stage's codes into the bf16 W tile (value = bf16(scale * (code - 8)), laid
// out as the SWIZZLE_128B tile TMA would have written) before the MMA reads it.
template <int kNT, bool kW4, int kAR>
__global__ void __launch_bounds__(kSmThreads, 1) small_m_kernel(const __grid_constant__ SmallMParams p) {
  using C = SmallMCfg<kNT, kW4, kAR>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wring = smem + S * C::kStageBytes;         // [kWBufs][16 KB] 4-bit: expanded W tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(wring + C::kWRingBytes + C::kBsBytes);
  uint64_t* full = bars;                 // [S]
  uint64_t* empty = bars + S;            // [S]
  uint64_t* wfull = bars + 2 * S;        // [kWBufs] 4-bit: W tile expanded (one arrival per epilogue warp)
  uint64_t* wempty = wfull + (kW4 ? C::kWBufs : 0);   // [kWBufs] 4-bit: W tile read by the MMAs
  uint64_t* acc_full = wempty + (kW4 ? C::kWBufs : 0);
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __nv_bfloat16* Bs = reinterpret_cast<__nv_bfloat16*>(wring + C::kWRingBytes);   // [F][r + 2], first in the tail
  float* Dp = reinterpret_cast<float*>(smem);                               // [128][kLd]  Z^T partial
  float* Tp = Dp + 128 * C::kLd;                                            // [128][kLd]  T^T partial
  float* Tf = Tp + 128 * C::kLd;                                            // [64][kNT]   summed T, tokens contiguous

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const int rank = static_cast<int>(cluster_ctarank());
  const int slice = blockIdx.x / p.splits;
  const int nkb = (p.d_in + 63) / 64;
  const int kb0 = rank * p.kb_per;
  const int kb1 = kb0 + p.kb_per < nkb ? kb0 + p.kb_per : nkb;
  const int nk = kb1 > kb0 ? kb1 - kb0 : 0;
  const int F = 128 / p.splits;          // features of the slice this CTA finishes
  const int f0 = rank * F;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < (kW4 ? C::kWBufs : 0); ++i) { mbar_init(&wfull[i], 4); mbar_init(&wempty[i], 1); }
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
  if (threadIdx.x == 0) {
    if constexpr (kW4) tma_prefetch_desc(&p.tm_ws);
    if (!kW4 || p.Wt == nullptr) tma_prefetch_desc(&p.tm_w);
    tma_prefetch_desc(&p.tm_a);
    tma_prefetch_desc(&p.tm_x);
  }
  grid_dep_wait();
  if (threadIdx.x == 0) sm_trace(p, kTrEntry);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last();     // X and A are re-read by every cluster
      // Every slice's CTA of the same rank reads the same A and X tiles; each
      // slice starts its K loop at a different stage (slice mod stages) so
      // that those reads spread over the L2 instead of converging on one tile.
      const int ns = (nk + C::kKPS - 1) / C::kKPS;      // stages: kKPS K blocks each, the last possibly fewer
      const int rot = ns > 0 ? slice % ns : 0;
      RingPos rp;
      for (int i = 0; i < ns; ++i) {
        if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        const int si = (i + rot) % ns;
        const int kbf = kb0 + si * C::kKPS;              // the stage's first K block
        const int nb = (nk - si * C::kKPS) < C::kKPS ? (nk - si * C::kKPS) : C::kKPS;
        // bytes: 3D boxes and the scales' box count all kKPS blocks (zero
        // fill past the tensor included); per-block 2D boxes and code tiles nb
        // (the 3D A box is kAR rows, zero past r, so that A tile j sits at
        // kAOff + j * kABox as the 2D boxes of a_rows rows put it)
        uint32_t tx = p.load3d ? static_cast<uint32_t>(C::kKPS * (C::kXBox + C::kABox))
                               : static_cast<uint32_t>(nb * (C::kXBox + p.a_rows * 128));
        if constexpr (kW4) tx += C::kKPS * C::kSBox + nb * C::kQBox;
        else tx += (p.load3d ? C::kKPS : nb) * C::kWBox;
        mbar_arrive_expect_tx(&full[rp.stage], tx);
        if (p.load3d) {
          tma_load_3d_hint(st + C::kXOff, &p.tm_x3, &full[rp.stage], 0, 0, kbf, pol_x);
          tma_load_3d_hint(st + C::kAOff, &p.tm_a3, &full[rp.stage], 0, 0, kbf, pol_x);
          if constexpr (!kW4) tma_load_3d(st + C::kWOff, &p.tm_w3, &full[rp.stage], 0, slice * 128, kbf);
        } else {
          for (int j = 0; j < nb; ++j) {
            const int k0 = (kbf + j) * 64;
            tma_load_2d_hint(st + C::kXOff + j * C::kXBox, &p.tm_x, &full[rp.stage], k0, 0, pol_x);
            tma_load_2d_hint(st + C::kAOff + j * C::kABox, &p.tm_a, &full[rp.stage], k0, 0, pol_x);
            if constexpr (!kW4) tma_load_2d(st + C::kWOff + j * C::kWBox, &p.tm_w, &full[rp.stage], k0, slice * 128);
          }
        }
        if constexpr (kW4) {
          if (p.Wt != nullptr)        // the stage's code tiles are contiguous in the tiled layout
            bulk_load_1d(st + C::kQOff, p.Wt + (static_cast<size_t>(slice) * nkb + kbf) * kW4TileBytes,
                         static_cast<uint32_t>(nb * kW4TileBytes), &full[rp.stage]);
          else
            for (int j = 0; j < nb; ++j)   // codes: (kbf + j) * 32 bytes into each row
              tma_load_2d(st + C::kQOff + j * C::kQBox, &p.tm_w, &full[rp.stage], (kbf + j) * 32, slice * 128);
          tma_load_2d(st + C::kSOff, &p.tm_ws, &full[rp.stage], slice * 128, kbf);   // scales of groups kbf ..
        }
        if (i == 0) sm_trace(p, kTrFirstIssue);
        if (i < kSmTraceStages) sm_trace(p, kSmTracePoints + i);
        rp.next(S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdZ = idesc_bf16(128, kNT, false, false);
      const uint32_t kIdT = idesc_bf16(128, p.a_rows, false, false);
      const int ns = (nk + C::kKPS - 1) / C::kKPS;
      const int rot = ns > 0 ? slice % ns : 0;          // the producer's stage order
      RingPos rp, wp;                   // wp: the 4-bit W tile ring
      bool ok = true;
      for (int i = 0; i < ns && ok; ++i) {
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
        tc_fence_after();
        if (i == 0) sm_trace(p, kTrFirstData);
        if (i < kSmTraceStages) sm_trace(p, kSmTracePoints + kSmTraceStages + i);
        const int si = (i + rot) % ns;
        const int nb = (nk - si * C::kKPS) < C::kKPS ? (nk - si * C::kKPS) : C::kKPS;
        const uint32_t sst = smem_u32(smem + rp.stage * C::kStageBytes);
        for (int j = 0; j < nb; ++j) {
          if constexpr (kW4) {
            if (!mbar_wait(&wfull[wp.stage], wp.phase, ctl)) { ok = false; break; }
            tc_fence_after();
          }
          const uint32_t sx = sst + C::kXOff + j * C::kXBox;
          const uint32_t sa = sst + C::kAOff + j * C::kABox;
          const uint32_t sw = kW4 ? smem_u32(wring + wp.stage * C::kWBox) : sst + C::kWOff + j * C::kWBox;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t dw = sdesc_sw128(sw + kk * 32, 16, 1024);
            const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t dx = sdesc_sw128(sx + kk * 32, 16, 1024);
            const uint32_t acc = (i == 0 && j == 0 && kk == 0) ? 0u : 1u;
            mma_bf16(tbase, dw, dx, kIdZ, acc);          // Z^T partial: 128 rows of W x tokens
            mma_bf16(tbase + kNT, dx, da, kIdT, acc);    // T partial: 128-row token window x rows of A
          }
          if constexpr (kW4) {            // this block's W tile is free once these MMAs retire
            mma_commit(&wempty[wp.stage]);
            wp.next(C::kWBufs);
          }
        }
        if (!ok) break;
        mma_commit(&empty[rp.stage]);
        rp.next(S);
      }
      if (ok && nk > 0) mma_commit(acc_full);
      // Teardown: every MMA issued here retires before TMEM is freed.
      mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait(mma_done, 0, quiet);
      sm_trace(p, kTrLastMma);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps (128 threads)
    const int et = threadIdx.x - 64;
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int lrow = q * 32 + lane;
    // this CTA's F rows of B (bf16, row stride r + 2), loaded during the K loop
    for (int i = et; i < F * p.r; i += 128) {
      const int fl = i / p.r, c = i - fl * p.r;
      const int n = slice * 128 + f0 + fl;
      Bs[fl * (p.r + 2) + c] = n < p.d_out ? p.B[static_cast<size_t>(n) * p.r + c] : __float2bfloat16_rn(0.0f);
    }
    if constexpr (kW4) {
      // Dequantise each K block's codes into the next W tile of the W ring:
      // thread lrow owns row lrow (32 bytes of codes, one scale) and writes
      // its 128-byte row of the SWIZZLE_128B tile, 16-byte chunk c (features
      // 8c .. 8c + 7) at position c ^ (lrow & 7).  Stages come in the
      // producer's order (rotated by slice).
      const int ns = (nk + C::kKPS - 1) / C::kKPS;
      const int rot = ns > 0 ? slice % ns : 0;
      RingPos rp, wp;
      const bool tr = p.trace != nullptr && et == 0;
      unsigned long long t_wait = 0, t_work = 0, t0 = tr ? sm_clock_ns() : 0;
      bool ok_dq = true;
      for (int i = 0; i < ns && ok_dq; ++i) {
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) break;
        const int si = (i + rot) % ns;
        const int nb = (nk - si * C::kKPS) < C::kKPS ? (nk - si * C::kKPS) : C::kKPS;
        const uint8_t* st = smem + rp.stage * C::kStageBytes;
        for (int j = 0; j < nb; ++j) {
          if (!mbar_wait(&wempty[wp.stage], wp.phase ^ 1u, ctl)) { ok_dq = false; break; }
          if (tr) { const unsigned long long t1 = sm_clock_ns(); t_wait += t1 - t0; t0 = t1; }
          const uint4* codes = reinterpret_cast<const uint4*>(st + C::kQOff + j * C::kQBox + lrow * 32);
          const uint4 c0 = codes[0], c1 = codes[1];
          const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const __nv_bfloat162 sc2 =
              __bfloat162bfloat162(reinterpret_cast<const __nv_bfloat16*>(st + C::kSOff + j * C::kSBox)[lrow]);
          uint4* wrow = reinterpret_cast<uint4*>(wring + wp.stage * C::kWBox + lrow * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) wrow[c ^ (lrow & 7)] = w4_word(words[c], sc2);
          fence_proxy_async_smem();     // the tensor core reads the tile through the async proxy
          __syncwarp();                 // the warp's rows are written; one arrival per warp
          if (lane == 0) mbar_arrive(&wfull[wp.stage]);
          if (tr) { const unsigned long long t1 = sm_clock_ns(); t_work += t1 - t0; t0 = t1; }
          wp.next(C::kWBufs);
        }
        rp.next(S);
      }
      if (tr) {
        p.trace[static_cast<size_t>(blockIdx.x) * kSmTraceStride + kTrDqWait] = t_wait;
        p.trace[static_cast<size_t>(blockIdx.x) * kSmTraceStride + kTrDqWork] = t_work;
      }
    }
    bool got = true;
    if (nk > 0) got = mbar_wait(acc_full, 0, ctl);
    const bool ok = bar_sync_and<1, 128>(got);
    // the T partial's lanes are tokens: only the first kNT are real (a
    // warp-uniform test); each such thread parks its token's r values
    // transposed, Tp[c][token], the layout the cluster sum below reads
    const bool t_rows = q * 32 < kNT;
    float4* drow = reinterpret_cast<float4*>(Dp + lrow * C::kLd);
    const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);
    if (ok && t_rows) {
      if (nk > 0) {
        tc_fence_after();
        for (int c0 = 0; c0 < p.a_rows; c0 += 16) {
          float t[16];
          tmem_ld16f(tl + static_cast<uint32_t>(kNT + c0), t);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c0 + c < p.r) Tp[(c0 + c) * C::kLd + lrow] = t[c];
        }
      } else {
        for (int c = 0; c < p.r; ++c) Tp[c * C::kLd + lrow] = 0.0f;
      }
    }
    if (ok) {
      // Z partial of feature row lrow
      if (nk > 0) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < kNT; c0 += 16) {
          float v[16];
          tmem_ld16f(tl + static_cast<uint32_t>(c0), v);
#pragma unroll
          for (int c = 0; c < 16; c += 4) drow[(c0 + c) / 4] = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kNT / 4; ++c) drow[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
    if (et == 0) sm_trace(p, kTrPublished);
  }
  tc_fence_before();
  __syncwarp();   // the cluster barrier is .aligned: each warp arrives converged
  // every CTA of the cluster has parked its partials
  cluster_sync_all();

  if (warp >= 2 && *abort_flag == 0u) {
    const int et = threadIdx.x - 64;
    if (et == 0) sm_trace(p, kTrSynced);
    const uint32_t dp_addr = smem_u32(Dp), tp_addr = smem_u32(Tp);
    const int M4 = (p.M + 3) >> 2;          // token quads (rows >= M hold zeros)
    const int nz = F * M4;                  // Z items: (feature, token quad)
    // Issue the peers' loads of this thread's first Z item now, so that their
    // latency overlaps the T sum below; they are summed after it.
    float4 zv[kSmMaxCluster];
    if (et < nz) {
      const int fl = et / M4, m0 = (et - fl * M4) * 4;
      const uint32_t a = dp_addr + static_cast<uint32_t>(((f0 + fl) * C::kLd + m0) * 4);
#pragma unroll
      for (int qq = 0; qq < kSmMaxCluster; ++qq)
        if (qq < p.splits) zv[qq] = ld_dsmem_f32x4(mapa_shared(a, static_cast<uint32_t>(qq)));
    }
    // T[m][c] = sum over the cluster's ranks (in order) of T^T[c][m], 4 tokens at a time
    for (int i = et; i < p.r * M4; i += 128) {
      const int c = i / M4, m0 = (i - c * M4) * 4;
      const float4 t = cluster_sum4(tp_addr + static_cast<uint32_t>((c * C::kLd + m0) * 4), p.splits);
      reinterpret_cast<float4*>(Tf)[(c * kNT + m0) / 4] = t;
      if (slice == 0 && rank == 0 && p.T_save != nullptr) {
        const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (m0 + j < p.M) p.T_save[static_cast<size_t>(m0 + j) * p.r + c] = tv[j];
      }
    }
    bar_sync_named<1, 128>();
    if (et == 0) sm_trace(p, kTrTSummed);
    // this CTA's features [f0, f0 + F) of the slice, 4 tokens per item
    for (int i = et; i < nz; i += 128) {
      const int fl = i / M4, m0 = (i - fl * M4) * 4;   // consecutive threads: consecutive quads of a row
      const int n = slice * 128 + f0 + fl;
      float4 zs;
      if (i == et) {
        zs = zv[0];
#pragma unroll
        for (int qq = 1; qq < kSmMaxCluster; ++qq)
          if (qq < p.splits) { zs.x += zv[qq].x; zs.y += zv[qq].y; zs.z += zv[qq].z; zs.w += zv[qq].w; }
      } else {
        zs = cluster_sum4(dp_addr + static_cast<uint32_t>(((f0 + fl) * C::kLd + m0) * 4), p.splits);
      }
      float z[4] = {zs.x, zs.y, zs.z, zs.w};
      float lora[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const __nv_bfloat16* brow = Bs + fl * (p.r + 2);
      const float4* tcol = reinterpret_cast<const float4*>(Tf) + m0 / 4;
      for (int c = 0; c < p.r; ++c) {
        const float b = __bfloat162float(brow[c]);
        const float4 t = tcol[c * (kNT / 4)];
        lora[0] = fmaf(b, t.x, lora[0]);
        lora[1] = fmaf(b, t.y, lora[1]);
        lora[2] = fmaf(b, t.z, lora[2]);
        lora[3] = fmaf(b, t.w, lora[3]);
      }
      if (n < p.d_out) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = m0 + j;
          if (m >= p.M) break;
          float v = fmaf(p.s, lora[j], z[j]);
          if (p.act == LORA_ACT_SILU) {
            if (p.Z_save != nullptr) p.Z_save[static_cast<size_t>(m) * p.d_out + n] = v;
            v = v / (1.0f + expf(-v));
          }
          p.Y[static_cast<size_t>(m) * p.d_out + n] = __float2bfloat16_rn(v);
        }
      }
    }
    if (et == 0) sm_trace(p, kTrCombined);
  }
  // peers may still read this CTA's shared memory until every CTA is done
  __syncwarp();
  cluster_sync_all();
  if (threadIdx.x == 0) sm_trace(p, kTrExit);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <int kNT, bool kW4, int kAR>
cudaError_t launch_small_m_kernel(const SmallMParams& p, int slices, bool pdl, cudaStream_t st) {
  using C = SmallMCfg<kNT, kW4, kAR>;
  auto k = small_m_kernel<kNT, kW4, kAR>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(slices * p.splits), 1, 1);
  cfg.blockDim = dim3(kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}

// Cluster size: the largest power of two (<= 16, <= the K blocks) with which
// all slices' clusters are resident at once (the device's answer for this
// kernel, shared memory and cluster shape), so the launch is a single wave.
template <int kNT, bool kW4, int kAR>
int small_m_splits_t(int slices, int nkb) {
  using C = SmallMCfg<kNT, kW4, kAR>;
  auto k = small_m_kernel<kNT, kW4, kAR>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  int best = 1;
  for (int s = 2; s <= kSmMaxCluster && s <= nkb; s *= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(slices * s), 1, 1);
    cfg.blockDim = dim3(kSmThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(s);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    if (n < slices) break;
    best = s;
  }
  return best;
}

// A-slot rows reserved per K block: 16 (r <= 16) or 64 (r <= 64).
inline int small_m_ar(int64_t r) { return r <= 16 ? 16 : 64; }

template <bool kW4, int kAR>
int small_m_splits_ar(int nt, int slices, int nkb) {
  if (nt == 16) return small_m_splits_t<16, kW4, kAR>(slices, nkb);
  if (nt == 32) return small_m_splits_t<32, kW4, kAR>(slices, nkb);
  return small_m_splits_t<64, kW4, kAR>(slices, nkb);
}

inline int small_m_splits(int nt, bool w4, int64_t r, int64_t d_in, int64_t d_out) {
  const int slices = static_cast<int>((d_out + 127) / 128);
  const int nkb = static_cast<int>((d_in + 63) / 64);
  const bool a16 = small_m_ar(r) == 16;
  if (w4) return a16 ? small_m_splits_ar<true, 16>(nt, slices, nkb) : small_m_splits_ar<true, 64>(nt, slices, nkb);
  return a16 ? small_m_splits_ar<false, 16>(nt, slices, nkb) : small_m_splits_ar<false, 64>(nt, slices, nkb);
}

template <bool kW4, int kAR>
cudaError_t launch_small_m_ar(const SmallMParams& p, int nt, int slices, bool pdl, cudaStream_t st) {
  if (nt == 16) return launch_small_m_kernel<16, kW4, kAR>(p, slices, pdl, st);
  if (nt == 32) return launch_small_m_kernel<32, kW4, kAR>(p, slices, pdl, st);
  return launch_small_m_kernel<64, kW4, kAR>(p, slices, pdl, st);
}

inline cudaError_t launch_small_m(const SmallMParams& p, int nt, bool w4, int slices, bool pdl, cudaStream_t st) {
  const bool a16 = small_m_ar(p.r) == 16;
  if (w4) return a16 ? launch_small_m_ar<true, 16>(p, nt, slices, pdl, st) : launch_small_m_ar<true, 64>(p, nt, slices, pdl, st);
  return a16 ? launch_small_m_ar<false, 16>(p, nt, slices, pdl, st)
             : launch_small_m_ar<false, 64>(p, nt, slices, pdl, st);
}

}  // namespace lora
