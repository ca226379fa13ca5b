// lora_small_m.cuh — forward for few tokens (M <= 64).  With so few tokens the
// layer is bound by reading W once from HBM (2 M d_in d_out FLOP on about
// 2 d_in d_out bytes), so the kernel is laid out for bandwidth.
//
// The rows of A are treated as one more 128-row slice in front of W's slices:
// streaming [A ; W] against X gives [T^T ; Z_main^T] in one pass, so T = X A^T
// costs no separate kernel, no extra CTAs and no dependent round trips while
// the memory system is busy with W.  Slice 0 (A, r rows, zero-filled to 128 by
// the TMA box) has almost no DRAM traffic and finishes first.
//
// One cooperative grid of at most one CTA per SM, stream-K over units of
// (128-row slice x 128-wide K chunk), slice-major, cut into equal contiguous
// runs (one per CTA).  Per unit one TMA stage brings two 64-wide boxes of the
// slice and the matching X boxes (M tokens, zero-filled to kNT rows); the MMA
// warp accumulates [128 rows x kNT tokens] in tensor memory (swap-AB: the
// weight rows are the M-side operand), double-buffered across segments.  When
// a CTA's part of a slice ends, its fp32 partial goes to global memory and the
// CTA bumps the slice's arrival counter; the CTA that arrives last (it learns
// so from the counter, without waiting) sums the slice's partials in slot
// order and finishes the slice:
//   slice 0:  T (and T_save) from rows < r, then a release of the T-ready flag;
//   slice s:  after a bounded wait for T-ready (set long before, in practice),
//             Z = partial sum + s T B^T, activation, Y.
// The cooperative launch guarantees that every CTA is resident, so the wait
// for the slice-0 CTAs always ends.  The counters live in the workspace header
// and are zero at rest: the calls that use them put them back to zero.
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
  float* t_buf;              // [M x r] T, written by slice 0's combiner
  float* d_part;             // [slices][max_seg][128 x kNT] partials ([A ; W] slices)
  uint32_t* counters;        // [slices] arrivals, then t_ready, slices_done (zero at rest)
  uint32_t* status;
  int M, d_in, d_out, r;
  float s;
  int act;
  int slices, nkc;           // 128-row slices of [A ; W] (1 + ceil(d_out / 128)); 128-wide K chunks
  int run;                   // units per CTA
  int max_seg;               // partial slots per slice
  unsigned long long* trace; // null, or [grid][kSmTracePoints] globaltimer stamps (debugging)
};

// Trace points of one CTA (LORA_LINEAR_DEBUG=2 prints them per launch).
enum SmTrace : int {
  kTrEntry = 0, kTrFirstIssue, kTrFirstData, kTrLastMma, kTrPublished, kTrCombined, kTrExit, kSmTracePoints
};

__device__ __forceinline__ void sm_trace(const SmallMParams& p, int point) {
  if (p.trace != nullptr) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
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

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
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
  float* Ts = reinterpret_cast<float*>(smem + S * C::kStageBytes + 1024);   // T [kNT x 64]

  uint32_t* t_ready = p.counters + p.slices;
  uint32_t* slices_done = p.counters + p.slices + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const int w = blockIdx.x;
  const int units = p.slices * p.nkc;
  const int u0 = w * p.run;
  const int u1 = u0 + p.run < units ? u0 + p.run : units;
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
  if (threadIdx.x == 0) sm_trace(p, kTrEntry);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last();     // X is re-read by every CTA
      RingPos rp;
      for (int u = u0; u < u1; ++u) {
        if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        const int slice = u / p.nkc;
        const int k0 = (u - slice * p.nkc) * 128;
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
        if (u == u0) sm_trace(p, kTrFirstIssue);
        rp.next(S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, kNT, false, false);
      RingPos rp;
      int seg = 0;
      bool first = true;
      for (int u = u0; u < u1; ++u) {
        const int slice = u / p.nkc;
        const uint32_t buf = seg & 1;
        if (first) {
          // a new segment: its accumulator buffer must have been read out
          if (!mbar_wait(&seg_empty[buf], ((seg >> 1) & 1) ^ 1u, ctl)) break;
          tc_fence_after();
        }
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) break;
        tc_fence_after();
        if (u == u0) sm_trace(p, kTrFirstData);
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
        if (u + 1 == u1 || (u + 1) / p.nkc != slice) {
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
    int u = u0;
    bool have_t = false;                    // T staged in shared memory
    while (u < u1) {
      const int slice = u / p.nkc;
      const int ue = (slice + 1) * p.nkc < u1 ? (slice + 1) * p.nkc : u1;
      const uint32_t buf = seg & 1;
      const bool got = mbar_wait(&seg_full[buf], (seg >> 1) & 1, ctl);
      if (!bar_sync_and<1, 128>(got)) break;        // all epilogue threads leave together
      tc_fence_after();
      // CTAs w_first..w_last share this slice; this CTA's partial goes to slot w - w_first
      const int w_first = (slice * p.nkc) / p.run;
      const int w_last = (slice * p.nkc + p.nkc - 1) / p.run;
      float* dst = p.d_part + ((static_cast<size_t>(slice) * p.max_seg + (w - w_first)) * 128 + lrow) * kNT;
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
      u = ue;
      // publish the partial; the CTA that completes the slice combines it
      __threadfence();
      bar_sync_named<1, 128>();
      if (et == 0) {
        const uint32_t arrived = atomicAdd(&p.counters[slice], 1u) + 1u;
        *last_flag = arrived == static_cast<uint32_t>(w_last - w_first + 1) ? 1 : 0;
      }
      bar_sync_named<1, 128>();
      if (et == 0) sm_trace(p, kTrPublished);
      if (*last_flag == 0) continue;
      __threadfence();
      // ---- combine: the slice's partials in slot order
      const int nseg = w_last - w_first + 1;
      float z[kNT];
#pragma unroll
      for (int m = 0; m < kNT; ++m) z[m] = 0.0f;
      constexpr int kSegUnroll = kNT <= 16 ? 4 : (kNT <= 32 ? 2 : 1);   // partial loads in flight
#pragma unroll kSegUnroll
      for (int sg = 0; sg < nseg; ++sg) {
        const float4* src =
            reinterpret_cast<const float4*>(p.d_part + ((static_cast<size_t>(slice) * p.max_seg + sg) * 128 + lrow) * kNT);
#pragma unroll
        for (int m4 = 0; m4 < kNT / 4; ++m4) {
          const float4 v = __ldcg(src + m4);
          z[4 * m4] += v.x;
          z[4 * m4 + 1] += v.y;
          z[4 * m4 + 2] += v.z;
          z[4 * m4 + 3] += v.w;
        }
      }
      if (slice == 0) {
        // rows < r hold T^T: T[m][lrow] for the M real tokens
        if (lrow < p.r) {
#pragma unroll
          for (int m = 0; m < kNT; ++m) {
            if (m < p.M) {
              __stcg(p.t_buf + static_cast<size_t>(m) * p.r + lrow, z[m]);
              if (p.T_save != nullptr) p.T_save[static_cast<size_t>(m) * p.r + lrow] = z[m];
            }
          }
        }
        __threadfence();
        bar_sync_named<1, 128>();
        if (et == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(t_ready), "r"(1u) : "memory");
      } else {
        if (!have_t) {
          // T-ready was released by slice 0's combiner, normally long ago
          if (et == 0) {
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
          bar_sync_named<1, 128>();
          have_t = true;
        }
        const int n = (slice - 1) * 128 + lrow;
        if (n < p.d_out) {
#pragma unroll 8
          for (int c = 0; c < p.r; ++c) {
            const float b = p.s * __bfloat162float(p.B[static_cast<size_t>(n) * p.r + c]);
#pragma unroll
            for (int m = 0; m < kNT; ++m) z[m] = fmaf(b, Ts[m * 64 + c], z[m]);
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
      }
      if (et == 0) {
        sm_trace(p, kTrCombined);
        p.counters[slice] = 0u;        // back to zero for the next call
        const uint32_t done = atomicAdd(slices_done, 1u) + 1u;
        if (done == static_cast<uint32_t>(p.slices)) {
          // every slice is finished: slice 0 has released T and every other
          // combiner has passed its wait for it
          *slices_done = 0u;
          *t_ready = 0u;
        }
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
cudaError_t launch_small_m_kernel(const SmallMParams& p, int grid, cudaStream_t st) {
  using C = SmallMCfg<kNT>;
  auto k = small_m_kernel<kNT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs co-resident: a combiner may wait for slice 0
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}

// Work split for a grid of at most `grid` CTAs: slices of [A ; W], units of
// 128 K columns, equal contiguous runs.
struct SmallMSplit {
  int slices = 0, nkc = 0, run = 0, n_w = 0, max_seg = 0;
};

inline SmallMSplit small_m_split(int64_t d_in, int64_t d_out, int grid) {
  SmallMSplit s;
  s.slices = 1 + static_cast<int>((d_out + 127) / 128);
  s.nkc = static_cast<int>((d_in + 127) / 128);
  const int units = s.slices * s.nkc;
  s.run = (units + grid - 1) / grid;
  s.n_w = (units + s.run - 1) / s.run;
  for (int sl = 0; sl < s.slices; ++sl) {
    const int seg = (sl * s.nkc + s.nkc - 1) / s.run - (sl * s.nkc) / s.run + 1;
    if (seg > s.max_seg) s.max_seg = seg;
  }
  return s;
}

inline cudaError_t launch_small_m(const SmallMParams& p, int nt, int grid, cudaStream_t st) {
  if (nt == 16) return launch_small_m_kernel<16>(p, grid, st);
  if (nt == 32) return launch_small_m_kernel<32>(p, grid, st);
  return launch_small_m_kernel<64>(p, grid, st);
}

}  // namespace lora
