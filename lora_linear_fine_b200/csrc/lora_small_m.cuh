// lora_small_m.cuh — forward for few tokens (M <= 64).  With so few tokens the
// layer is bound by reading W once from HBM (2 M d_in d_out FLOP on about
// 2 d_in d_out bytes), so the kernel is laid out for bandwidth.
//
// The rows of A are streamed like one more 128-row slice of weights ("slice
// 0", in front of W's slices 1..): [A ; W] against X gives [T^T ; Z_main^T] in
// one pass, so T = X A^T needs no kernel of its own.  Slice 0's K chunks are
// spread one per CTA as the first unit of CTAs 0, 1, ... (A has r rows, so a
// chunk costs almost no DRAM traffic): T is complete about one unit into the
// pass, long before any slice of W.
//
// One cooperative grid of at most one CTA per SM.  W's units (128-row slice x
// 128-wide K chunk, slice-major) are cut into equal contiguous runs, one per
// CTA.  Per unit one TMA stage brings two 64-wide boxes of the slice and the
// matching X boxes (M tokens, zero-filled to kNT rows); the MMA warp
// accumulates [128 rows x kNT tokens] in tensor memory (swap-AB: the weight
// rows are the M-side operand), double-buffered across segments.  When a
// CTA's part of a slice ends, its fp32 partial goes to global memory and the
// CTA bumps the slice's arrival counter; the CTA whose arrival completes the
// slice (it learns so from the counter value) finishes it:
//   slice 0: sums the partials in slot order, writes T (and T_save) from
//     rows < r, and releases the T-ready flag;
//   a slice of W: sums the partials in slot order (deterministic), adds
//     s T B^T, applies the activation and stores Y.  It needs T: T is ready
//     about one unit into the pass, so the bounded wait for the flag is
//     normally already over; the cooperative launch makes every CTA resident,
//     so the wait always ends.
// The counters live in the workspace header and are zero at rest: the last
// finisher of a call puts them back to zero.
#pragma once

#include <cuda_runtime.h>

#include "lora_linear.h"
#include "sm100.cuh"

namespace lora {

constexpr int64_t kSmallMMax = 64;
constexpr int kSmThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

struct SmallMParams {
  CUtensorMap tm_w;          // W [d_out x d_in], box 64 x 128
  CUtensorMap tm_a;          // A [r x d_in],     box 64 x 128 (rows >= r zero-filled)
  CUtensorMap tm_x;          // X [M x d_in],     box 64 x kNT (rows >= M zero-filled)
  const __nv_bfloat16* B;    // [d_out x r]
  __nv_bfloat16* Y;          // [M x d_out]
  float* T_save;             // [M x r] or null
  float* Z_save;             // [M x d_out] or null (SiLU)
  float* t_buf;              // [M x r] T, written by slice 0's finisher
  float* d_part0;            // [nseg0][128 x kNT] slice-0 partials
  float* d_part;             // [wslices][max_seg][128 x kNT] partials of W's slices
  uint32_t* counters;        // [1 + wslices] arrivals, then T-ready, finished slices (zero at rest)
  uint32_t* status;
  int M, d_in, d_out, r;
  float s;
  int act;
  int wslices, nkc;          // 128-row slices of W; 128-wide K chunks
  int run;                   // W units per CTA
  int grid;                  // CTAs
  int nseg0;                 // CTAs holding slice-0 chunks: min(nkc, grid)
  int max_seg;               // partial slots per slice of W
  unsigned long long* trace; // null, or [grid][kSmTracePoints] globaltimer stamps (debugging)
};

// Trace points of one CTA (LORA_LINEAR_DEBUG=2 prints them per launch).
enum SmTrace : int {
  kTrEntry = 0, kTrFirstIssue, kTrFirstData, kTrLastMma, kTrPublished, kTrCombined, kTrExit, kSmTracePoints
};

__device__ __forceinline__ void sm_trace(const SmallMParams& p, int point) {
  if (p.trace != nullptr) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t) : : "memory");
    p.trace[static_cast<size_t>(blockIdx.x) * kSmTracePoints + point] = t;
  }
}

template <int kNT>
struct SmallMCfg {
  static constexpr int kWBox = 128 * 64 * 2;            // one weight box: 128 rows x 64
  static constexpr int kXBox = kNT * 64 * 2;            // one X box: kNT rows x 64
  static constexpr int kStageBytes = 2 * kWBox + 2 * kXBox;
  static constexpr int kTailBytes = 1024 + kNT * 64 * 4 + 1024;   // barriers, T tile, alignment slack
  static constexpr int kStages0 = (kSmemLimitBytes - kTailBytes) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kTailBytes;
  static constexpr uint32_t kTmemCols = (2 * kNT) <= 32 ? 32 : ((2 * kNT) <= 64 ? 64 : 128);
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kStages >= 3, "ring too shallow");
};

// The units of CTA w, in order: its slice-0 chunks w, w + grid, ... (< nkc),
// then its run of W units.
struct SmUnits {
  int na;    // slice-0 chunks
  int uw0;   // first W unit
  int n;     // units in all
  __device__ __forceinline__ SmUnits(const SmallMParams& p, int w) {
    na = w < p.nkc ? (p.nkc - 1 - w) / p.grid + 1 : 0;
    const int total_w = p.wslices * p.nkc;
    uw0 = w * p.run;
    const int uw1 = uw0 + p.run < total_w ? uw0 + p.run : total_w;
    n = na + (uw1 > uw0 ? uw1 - uw0 : 0);
  }
  // slice (0 = A, s >= 1 = W rows [128 (s - 1), +128)) and K chunk of unit i
  __device__ __forceinline__ void at(const SmallMParams& p, int w, int i, int& slice, int& kc) const {
    if (i < na) {
      slice = 0;
      kc = w + i * p.grid;
    } else {
      const int u = uw0 + (i - na);
      slice = 1 + u / p.nkc;
      kc = u - (slice - 1) * p.nkc;
    }
  }
};

__device__ __forceinline__ int small_m_first_cta(const SmallMParams& p, int slice) {
  return ((slice - 1) * p.nkc) / p.run;
}
__device__ __forceinline__ int small_m_nseg(const SmallMParams& p, int slice) {
  if (slice == 0) return p.nseg0;
  return ((slice - 1) * p.nkc + p.nkc - 1) / p.run - small_m_first_cta(p, slice) + 1;
}
// Arrivals that finish a slice: one per CTA holding part of it.
__device__ __forceinline__ uint32_t small_m_target(const SmallMParams& p, int slice) {
  return static_cast<uint32_t>(small_m_nseg(p, slice));
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// A slice is finished: count it; the last finisher of the call resets the
// shared words (every finisher of W has passed its wait for T by then).
__device__ __forceinline__ void small_m_slice_done(const SmallMParams& p, int slice) {
  uint32_t* t_ready = p.counters + 1 + p.wslices;
  uint32_t* done = t_ready + 1;
  p.counters[slice] = 0u;
  if (atomicAdd(done, 1u) + 1u == static_cast<uint32_t>(1 + p.wslices)) {
    *done = 0u;
    *t_ready = 0u;
  }
}
__device__ __forceinline__ float* small_m_slot(const SmallMParams& p, int slice, int slot, int lrow, int nt) {
  if (slice == 0) return p.d_part0 + (static_cast<size_t>(slot) * 128 + lrow) * nt;
  return p.d_part + ((static_cast<size_t>(slice - 1) * p.max_seg + slot) * 128 + lrow) * nt;
}

// Sum of a slice's partials for row lrow, in slot order.
template <int kNT>
__device__ __forceinline__ void small_m_sum_partials(const SmallMParams& p, int slice, int lrow, float (&z)[kNT]) {
  const int nseg = small_m_nseg(p, slice);
#pragma unroll
  for (int m = 0; m < kNT; ++m) z[m] = 0.0f;
  constexpr int kSegUnroll = kNT <= 16 ? 4 : (kNT <= 32 ? 2 : 1);   // partial loads in flight
#pragma unroll kSegUnroll
  for (int sg = 0; sg < nseg; ++sg) {
    const float4* src = reinterpret_cast<const float4*>(small_m_slot(p, slice, sg, lrow, kNT));
#pragma unroll
    for (int m4 = 0; m4 < kNT / 4; ++m4) {
      const float4 v = __ldcg(src + m4);
      z[4 * m4] += v.x;
      z[4 * m4 + 1] += v.y;
      z[4 * m4 + 2] += v.z;
      z[4 * m4 + 3] += v.w;
    }
  }
}

// Finish slice 0 (all 128 epilogue threads): T[m][c] = sum over the slice-0
// partials, in slot order, of row c (< r), column m (< M).  One element per
// thread at a time with 16 partial loads in flight.
template <int kNT>
__device__ __forceinline__ void small_m_finish_t(const SmallMParams& p, int et) {
  const int ne = p.r * p.M;
  const size_t stride = static_cast<size_t>(128) * kNT;     // between slots
  for (int e = et; e < ne; e += 128) {
    const int row = e / p.M, m = e - row * p.M;
    const float* src = p.d_part0 + static_cast<size_t>(row) * kNT + m;
    float acc = 0.0f;
    for (int s0 = 0; s0 < p.nseg0; s0 += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = s0 + u < p.nseg0 ? __ldcg(src + (s0 + u) * stride) : 0.0f;
#pragma unroll
      for (int u = 0; u < 16; ++u) acc += v[u];                // slot order; + 0 past the last slot
    }
    __stcg(p.t_buf + static_cast<size_t>(m) * p.r + row, acc);
    if (p.T_save != nullptr) p.T_save[static_cast<size_t>(m) * p.r + row] = acc;
  }
}

// Finish a slice of W (all 128 epilogue threads): Z = partial sum + s T B^T,
// activation, Y (and Z_save).  T, this thread's row of B and the partials are
// all requested before the first use.
template <int kNT>
__device__ __forceinline__ void small_m_finish_slice(const SmallMParams& p, int slice, int et, int lrow, float* Ts) {
  const int n = (slice - 1) * 128 + lrow;
  if (et == 0) {
    const uint32_t* t_ready = p.counters + 1 + p.wslices;
    const long long t0 = clock64();
    while (ld_acquire_gpu(t_ready) == 0u) {
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicOr(p.status, kStatusWaitTimeout);
        break;
      }
    }
  }
  bar_sync_named<1, 128>();
  __threadfence();
#pragma unroll
  for (int k = 0; k < kNT / 2; ++k) {
    const int i = et + 128 * k;
    const int m = i >> 6, c = i & 63;
    Ts[i] = (m < p.M && c < p.r) ? __ldcg(p.t_buf + m * p.r + c) : 0.0f;
  }
  // B row prefetched in registers only while they are plentiful (kNT = 16)
  constexpr int kBq = kNT <= 16 ? 8 : 1;
  uint4 bq[kBq];
#pragma unroll
  for (int c8 = 0; c8 < kBq; ++c8)
    bq[c8] = (c8 * 8 < p.r && n < p.d_out)
                 ? __ldg(reinterpret_cast<const uint4*>(p.B + static_cast<size_t>(n) * p.r + c8 * 8))
                 : make_uint4(0u, 0u, 0u, 0u);
  float z[kNT];
  small_m_sum_partials<kNT>(p, slice, lrow, z);
  bar_sync_named<1, 128>();                 // T in shared memory
  if (n < p.d_out) {
#pragma unroll(kBq)
    for (int c8 = 0; c8 < 8; ++c8) {
      if (c8 * 8 < p.r) {
        uint4 bv;
        if constexpr (kBq == 8) bv = bq[c8];
        else bv = __ldg(reinterpret_cast<const uint4*>(p.B + static_cast<size_t>(n) * p.r + c8 * 8));
        const __nv_bfloat16* b8 = reinterpret_cast<const __nv_bfloat16*>(&bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float b = p.s * __bfloat162float(b8[e]);
#pragma unroll
          for (int m = 0; m < kNT; ++m) z[m] = fmaf(b, Ts[m * 64 + c8 * 8 + e], z[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kNT; ++m) {
      if (m < p.M) {
        float y = z[m];
        if (p.act == LORA_ACT_SILU) {
          if (p.Z_save != nullptr) p.Z_save[static_cast<size_t>(m) * p.d_out + n] = y;
          y = y / (1.0f + expf(-y));
        }
        p.Y[static_cast<size_t>(m) * p.d_out + n] = __float2bfloat16_rn(y);
      }
    }
  }
  bar_sync_named<1, 128>();                 // Ts is reused by the next finish
  if (et == 0) {
    sm_trace(p, kTrCombined);
    small_m_slice_done(p, slice);
  }
}

template <int kNT>
__global__ void __launch_bounds__(kSmThreads, 1) small_m_kernel(const __grid_constant__ SmallMParams p) {
  using C = SmallMCfg<kNT>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* full = bars;                 // [S]
  uint64_t* empty = bars + S;            // [S]
  uint64_t* seg_full = bars + 2 * S;     // [2] accumulator buffer b holds a finished segment
  uint64_t* seg_empty = seg_full + 2;    // [2] accumulator buffer b has been read out
  uint64_t* mma_done = seg_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(seg_full + 5);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* Ts = reinterpret_cast<float*>(smem + S * C::kStageBytes + 1024);                // T [kNT x 64]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const int w = blockIdx.x;
  const SmUnits units(p, w);
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&seg_full[b], 1); mbar_init(&seg_empty[b], 128); }
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  grid_dep_wait();
  if (threadIdx.x == 0) sm_trace(p, kTrEntry);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last();     // X is re-read by every CTA
      RingPos rp;
      for (int i = 0; i < units.n; ++i) {
        if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        int slice, kc;
        units.at(p, w, i, slice, kc);
        const int k0 = kc * 128;
        mbar_arrive_expect_tx(&full[rp.stage], C::kStageBytes);
        if (slice == 0) {
          tma_load_2d(st, &p.tm_a, &full[rp.stage], k0, 0);
          tma_load_2d(st + C::kWBox, &p.tm_a, &full[rp.stage], k0 + 64, 0);
        } else {
          tma_load_2d(st, &p.tm_w, &full[rp.stage], k0, (slice - 1) * 128);
          tma_load_2d(st + C::kWBox, &p.tm_w, &full[rp.stage], k0 + 64, (slice - 1) * 128);
        }
        tma_load_2d_hint(st + 2 * C::kWBox, &p.tm_x, &full[rp.stage], k0, 0, pol_x);
        tma_load_2d_hint(st + 2 * C::kWBox + C::kXBox, &p.tm_x, &full[rp.stage], k0 + 64, 0, pol_x);
        if (i == 0) sm_trace(p, kTrFirstIssue);
        rp.next(S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, kNT, false, false);
      RingPos rp;
      int seg = 0;
      bool first = true;
      for (int i = 0; i < units.n; ++i) {
        int slice, kc;
        units.at(p, w, i, slice, kc);
        const uint32_t buf = seg & 1;
        if (first) {
          // a new segment: its accumulator buffer must have been read out
          if (!mbar_wait(&seg_empty[buf], ((seg >> 1) & 1) ^ 1u, ctl)) break;
          tc_fence_after();
        }
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) break;
        tc_fence_after();
        if (i == 0) sm_trace(p, kTrFirstData);
        const uint32_t sw = smem_u32(smem + rp.stage * C::kStageBytes);
        const uint32_t sx = sw + 2 * C::kWBox;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t dw = sdesc_sw128(sw + (kk >> 2) * C::kWBox + (kk & 3) * 32, 16, 1024);
          const uint64_t dx = sdesc_sw128(sx + (kk >> 2) * C::kXBox + (kk & 3) * 32, 16, 1024);
          mma_bf16(tbase + buf * kNT, dw, dx, kId, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&empty[rp.stage]);
        rp.next(S);
        first = false;
        int next_slice = -1, next_kc = 0;
        if (i + 1 < units.n) units.at(p, w, i + 1, next_slice, next_kc);
        if (next_slice != slice) {
          mma_commit(&seg_full[buf]);
          ++seg;
          first = true;
        }
      }
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
    const int lrow = q * 32 + lane;         // row within the slice
    int seg = 0;
    int i = 0;
    while (i < units.n) {
      int slice, kc;
      units.at(p, w, i, slice, kc);
      // the segment runs while the slice stays the same
      int ie = i + 1;
      while (ie < units.n) {
        int s2, k2;
        units.at(p, w, ie, s2, k2);
        if (s2 != slice) break;
        ++ie;
      }
      const uint32_t buf = seg & 1;
      const bool got = mbar_wait(&seg_full[buf], (seg >> 1) & 1, ctl);
      if (!bar_sync_and<1, 128>(got)) break;        // all epilogue threads leave together
      tc_fence_after();
      const int slot = slice == 0 ? w : w - small_m_first_cta(p, slice);
      float* dst = small_m_slot(p, slice, slot, lrow, kNT);
      const uint32_t tl = tbase + buf * kNT + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < kNT; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tl + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          __stcg(reinterpret_cast<float4*>(dst + c0 + c),
                 make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2]),
                             __uint_as_float(v[c + 3])));
      }
      tc_fence_before();
      mbar_arrive(&seg_empty[buf]);
      ++seg;
      i = ie;
      // publish the partial; the arrival that completes the slice finishes it
      __threadfence();
      bar_sync_named<1, 128>();
      if (et == 0) {
        const uint32_t arrived = atomicAdd(&p.counters[slice], 1u) + 1u;
        *last_flag = arrived == small_m_target(p, slice) ? 1 : 0;
      }
      bar_sync_named<1, 128>();
      if (et == 0) sm_trace(p, kTrPublished);
      if (*last_flag == 0) continue;
      __threadfence();
      if (slice != 0) {
        small_m_finish_slice<kNT>(p, slice, et, lrow, Ts);
        continue;
      }
      // ---- slice 0: T = X A^T from rows < r, then the T-ready flag
      small_m_finish_t<kNT>(p, et);
      __threadfence();
      bar_sync_named<1, 128>();
      if (et == 0) {
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.counters + 1 + p.wslices), "r"(1u) : "memory");
        small_m_slice_done(p, 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) sm_trace(p, kTrExit);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <int kNT>
cudaError_t launch_small_m_kernel(const SmallMParams& p, cudaStream_t st) {
  using C = SmallMCfg<kNT>;
  auto k = small_m_kernel<kNT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid), 1, 1);
  cfg.blockDim = dim3(kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs resident: a finisher may wait for T
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}

// Work split for at most `grid` CTAs: W's units in equal contiguous runs,
// slice 0's K chunks one per CTA.
struct SmallMSplit {
  int wslices = 0, nkc = 0, run = 0, grid = 0, nseg0 = 0, max_seg = 0;
};

inline SmallMSplit small_m_split(int64_t d_in, int64_t d_out, int grid) {
  SmallMSplit s;
  s.wslices = static_cast<int>((d_out + 127) / 128);
  s.nkc = static_cast<int>((d_in + 127) / 128);
  const int units = s.wslices * s.nkc;
  s.run = (units + grid - 1) / grid;
  s.grid = (units + s.run - 1) / s.run;
  s.nseg0 = s.nkc < s.grid ? s.nkc : s.grid;
  for (int sl = 0; sl < s.wslices; ++sl) {
    const int seg = (sl * s.nkc + s.nkc - 1) / s.run - (sl * s.nkc) / s.run + 1;
    if (seg > s.max_seg) s.max_seg = seg;
  }
  return s;
}

inline cudaError_t launch_small_m(const SmallMParams& p, int nt, cudaStream_t st) {
  if (nt == 16) return launch_small_m_kernel<16>(p, st);
  if (nt == 32) return launch_small_m_kernel<32>(p, st);
  return launch_small_m_kernel<64>(p, st);
}

}  // namespace lora
