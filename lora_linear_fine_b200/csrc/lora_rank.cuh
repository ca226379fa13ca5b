// lora_rank.cuh — kernels for the rank-r side of the backward.
//
// rank_gemm_kernel: a split-K tcgen05 kernel for products whose result has
//   only r (<= 128) columns and whose reduction runs over tokens or features:
//     dA^T = X^T (s U)           [d_in  x r],  K = tokens   (X read MN-major)
//     dB   = dZ^T (s T)          [d_out x r],  K = tokens   (dZ read MN-major)
//     U_lo = dZ_lo B, T = X A^T  [M x r],      K = features (K-major)
//   The fp32-grade operands (s U, s T) are split into bf16 hi + lo parts and
//   summed as two MMAs into one fp32 accumulator, so the adapter gradients keep
//   fp32-grade precision although the tensor cores take bf16.
//   One CTA = one 128-row tile x one K range; it writes an fp32 partial that
//   reduce_partials_kernel sums in a fixed order (deterministic, no atomics).
// Also: the fixed-order reduction of split-K partials, the backward's
// preparation (B^T, transposed hi/lo s*T), the fp16 weight copy and the
// activation backward dZ = dY * act'(Z) as fp16 hi/lo.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace lora {

constexpr int kRankThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

// Where a finished rows x r rank result goes (any subset of the outputs):
//   f32  fp32, row-major [rows x r] (transpose_f32: [r x rows])
//   s16  bf16(scale * v), row-major [rows x r] (the LoRA K-block operand)
//   hi/lo  scale * v split into a 16-bit hi part and the rounded remainder,
//          transposed [r x ld] (bf16, or fp16 when hilo_f16)
struct RankOut {
  float* f32;
  int transpose_f32;
  __nv_bfloat16* s16;
  void* hi;
  void* lo;
  int ld;
  int hilo_f16;
  float scale;
  int rows, r;
};

__device__ __forceinline__ void emit_rank_row(const float* v, int row, const RankOut& o) {
  if (o.f32 != nullptr) {
    if (o.transpose_f32) {
      for (int c = 0; c < o.r; ++c) o.f32[static_cast<size_t>(c) * o.rows + row] = v[c];
    } else {
      float* d = o.f32 + static_cast<size_t>(row) * o.r;
      for (int c = 0; c < o.r; c += 4) *reinterpret_cast<float4*>(d + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    }
  }
  if (o.s16 != nullptr) {
    __nv_bfloat16* d = o.s16 + static_cast<size_t>(row) * o.r;
    for (int c = 0; c < o.r; c += 8) {
      uint4 pk;
      pk.x = pack_bf16x2(o.scale * v[c + 0], o.scale * v[c + 1]);
      pk.y = pack_bf16x2(o.scale * v[c + 2], o.scale * v[c + 3]);
      pk.z = pack_bf16x2(o.scale * v[c + 4], o.scale * v[c + 5]);
      pk.w = pack_bf16x2(o.scale * v[c + 6], o.scale * v[c + 7]);
      *reinterpret_cast<uint4*>(d + c) = pk;
    }
  }
  if (o.hi != nullptr) {
    for (int c = 0; c < o.r; ++c) {
      const float x = o.scale * v[c];
      const size_t i = static_cast<size_t>(c) * o.ld + row;
      if (o.hilo_f16) {
        const __half h = __float2half_rn(x);
        static_cast<__half*>(o.hi)[i] = h;
        static_cast<__half*>(o.lo)[i] = __float2half_rn(x - __half2float(h));
      } else {
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        static_cast<__nv_bfloat16*>(o.hi)[i] = h;
        static_cast<__nv_bfloat16*>(o.lo)[i] = __float2bfloat16_rn(x - __bfloat162float(h));
      }
    }
  }
}

struct RankGemmParams {
  CUtensorMap tm_a[2];
  CUtensorMap tm_b[2];
  // Dropout on the adapter input (K-major A = X only): keep bits of X, [rows x
  // mask_ld] bytes, bit j of byte b keeping element 8 b + j of a row; null for
  // none.  The epilogue warps zero the dropped elements of each stage's X
  // tiles in shared memory before the MMA warp reads them.
  const uint8_t* mask;
  int mask_ld;
  int rows;          // rows of the result (M side of the MMA)
  int K;             // reduction length
  int m_tiles;
  int kb_per_split;
  int npairs;        // products accumulated: sum over q < npairs of A[pa[q]] * B[pb[q]]
  int pa[4], pb[4];
  float* partial;    // [splits][m_tiles*128][RP] fp32; null when K is not split: results go to `out`
  RankOut out;
  uint32_t* status;
};

// kNA / kNB: number of distinct A / B operand tiles per stage (1 or 2).
// One pipeline stage covers kKS consecutive 64-wide K blocks: per A operand
// kKS K-major boxes of 128 rows x 64 (or two MN-major boxes of 64 x 64*kKS),
// per B operand kKS boxes of RP rows x 64.  Larger TMA boxes and several
// boxes per stage keep more DRAM traffic in flight per request (measured:
// 8 KB boxes stream at about half the rate of 32-64 KB stages).
// 64-wide K blocks per pipeline stage of rank_gemm_kernel: two for a single A
// operand of rank <= 64, else one (so that a stage stays within a quarter of
// shared memory).  The host sizes its TMA boxes and K splits with the same rule.
constexpr int rank_ks(int na, int rp) { return (na == 1 && rp <= 64) ? 2 : 1; }

template <bool kAMN, int kRP, int NA, int NB, bool kF16>
struct RankCfg {
  static constexpr int kNA = NA;
  static constexpr int kNB = NB;
  static constexpr int kKS = rank_ks(NA, kRP);             // 64-wide K blocks per stage
  static constexpr int kABytes = 128 * 64 * 2 * kKS;      // one A operand per stage
  static constexpr int kBBox = kRP * 128;                 // one B box (64 K)
  static constexpr int kBBytes = kBBox * kKS;             // one B operand per stage
  static constexpr int kStageBytes = kNA * kABytes + kNB * kBBytes;
  static constexpr int kStages0 = (kSmemLimitBytes - 2048) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + 2048;
  static constexpr uint32_t kTmemCols = kRP < 32 ? 32 : kRP;
};

template <bool kAMN, int kRP, int kNA, int kNB, bool kF16>
__global__ void __launch_bounds__(kRankThreads, 1) rank_gemm_kernel(const __grid_constant__ RankGemmParams p) {
  using C = RankCfg<kAMN, kRP, kNA, kNB, kF16>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* mma_done = acc_full + 1;
  uint64_t* masked = acc_full + 2;     // [S] dropout: the stage's X tiles are masked (one arrival per epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(masked + S);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const bool masking = !kAMN && p.mask != nullptr;
  const int mt = blockIdx.x % p.m_tiles;
  const int sp = blockIdx.x / p.m_tiles;
  constexpr int KS = C::kKS;
  const int nkb_all = (p.K + 64 * KS - 1) / (64 * KS);     // stages over the whole K
  const int kb0 = sp * p.kb_per_split;
  int kb1 = kb0 + p.kb_per_split;
  if (kb1 > nkb_all) kb1 = nkb_all;
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); mbar_init(&masked[i], 4); }
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
  grid_dep_wait();

  if (warp == 0) {
    if (lane == 0 && nkb > 0) {
      const uint64_t pol = l2_policy_evict_first();
      RingPos rp;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        uint64_t* fb = &full[rp.stage];
        mbar_arrive_expect_tx(fb, C::kStageBytes);
        const int k0 = (kb0 + i) * 64 * KS;
        const int m0 = mt * 128;
#pragma unroll
        for (int a = 0; a < C::kNA; ++a) {
          uint8_t* sa = st + a * C::kABytes;
          if constexpr (kAMN) {
            // two boxes of 64 rows-of-the-result x 64*KS K (tokens)
            tma_load_2d_hint(sa, &p.tm_a[a], fb, m0, k0, pol);
            tma_load_2d_hint(sa + C::kABytes / 2, &p.tm_a[a], fb, m0 + 64, k0, pol);
          } else {
#pragma unroll
            for (int kb = 0; kb < KS; ++kb) tma_load_2d_hint(sa + kb * 16384, &p.tm_a[a], fb, k0 + 64 * kb, m0, pol);
          }
        }
#pragma unroll
        for (int b = 0; b < C::kNB; ++b)
#pragma unroll
          for (int kb = 0; kb < KS; ++kb)
            tma_load_2d(st + C::kNA * C::kABytes + b * C::kBBytes + kb * C::kBBox, &p.tm_b[b], fb, k0 + 64 * kb, 0);
        rp.next(S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nkb > 0) {
      constexpr uint32_t kId = idesc_mma(128, kRP, kAMN, false, kF16);
      RingPos rp;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
        if (masking && !mbar_wait(&masked[rp.stage], rp.phase, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + rp.stage * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4 * KS; ++kk) {
          for (int pp = 0; pp < p.npairs; ++pp) {
            const uint32_t sa = st + p.pa[pp] * C::kABytes;
            const uint32_t sb = st + C::kNA * C::kABytes + p.pb[pp] * C::kBBytes + (kk >> 2) * C::kBBox;
            const uint64_t da = kAMN ? sdesc_sw128(sa + kk * 2048, C::kABytes / 2, 1024)
                                     : sdesc_sw128(sa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t db = sdesc_sw128(sb + (kk & 3) * 32, 16, 1024);
            mma_bf16(tbase, da, db, kId, (i == 0 && kk == 0 && pp == 0) ? 0u : 1u);
          }
        }
        mma_commit(&empty[rp.stage]);
        rp.next(S);
      }
      if (ok) mma_commit(acc_full);
      // Teardown: every MMA issued here retires before TMEM is freed.
      mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait(mma_done, 0, quiet);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    if (masking) {
      // Dropout: zero the dropped elements of each stage's X tiles.  Thread
      // `row` owns row `row` of every [128 x 64] SWIZZLE_128B box and its
      // 8 * KS keep bytes per stage, loaded one stage ahead so that their
      // latency hides behind the wait for the tiles.
      constexpr int kMB = 8 * KS;
      const int grow = mt * 128 + row;
      const bool in_rows = grow < p.rows;
      const uint8_t* mrow = p.mask + static_cast<size_t>(in_rows ? grow : 0) * p.mask_ld;
      const bool vec = (reinterpret_cast<uintptr_t>(p.mask) % kMB) == 0 && p.mask_ld % kMB == 0;
      uint32_t cur[kMB / 4], nxt[kMB / 4];
      if (nkb > 0) load_keep_bytes<kMB>(mrow, kb0 * kMB, p.mask_ld, in_rows, vec, cur);
      RingPos rp;
      for (int i = 0; i < nkb; ++i) {
        if (i + 1 < nkb) load_keep_bytes<kMB>(mrow, (kb0 + i + 1) * kMB, p.mask_ld, in_rows, vec, nxt);
        if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) break;
        uint8_t* st = smem + rp.stage * C::kStageBytes;
        mask_sw128_rows<KS>(st + row * 128, 16384, row, cur);
        fence_proxy_async_smem();     // the tensor core reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&masked[rp.stage]);
#pragma unroll
        for (int w = 0; w < kMB / 4; ++w) cur[w] = nxt[w];
        rp.next(S);
      }
    }
    float acc[kRP];
#pragma unroll
    for (int c = 0; c < kRP; ++c) acc[c] = 0.0f;
    bool have = nkb == 0;
    if (nkb > 0 && mbar_wait(acc_full, 0, ctl)) {
      have = true;
      tc_fence_after();
      __syncwarp();
      const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < kRP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tl + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c0 + c] = __uint_as_float(v[c]);
      }
    }
    if (have) {
      if (p.partial != nullptr) {
        float* dst = p.partial + (static_cast<size_t>(sp) * p.m_tiles * 128 + static_cast<size_t>(mt) * 128 + row) * kRP;
#pragma unroll
        for (int c = 0; c < kRP; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
      } else {
        const int grow = mt * 128 + row;
        if (grow < p.rows) emit_rank_row(acc, grow, p.out);
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

// Fixed-order sum of split-K partials for up to two independent jobs in one
// launch.
struct RankReduceJob {
  const float* partial;   // [splits][rows_pad][RP]
  int splits, rows_pad, RP;
  int rpb;                // result rows per block (1..kReduceRows): fewer rows, more blocks, for few rows
  RankOut out;
};

// Blocks of rpb (<= kReduceRows) result rows (grid-stride over row blocks;
// blockIdx.y selects the job).  Each thread sums float4 pieces of the partial
// rows over the splits in split order (eight splits of loads in flight; with
// few pieces and many splits, four threads per piece over quarters of the
// splits), into a shared-memory tile; then row-major outputs are written by warps along a
// row and transposed outputs by warps along a column, so every global access
// is coalesced and no index needs a division.  RP is a power of two and r a
// multiple of 8, so a float4 piece lies wholly inside or wholly past r.
constexpr int kReduceRows = 32;
constexpr int kMaxRank = 128;

__global__ void __launch_bounds__(256, 2) reduce_rank_kernel(RankReduceJob j0, RankReduceJob j1) {
  grid_dep_wait();
  const RankReduceJob& J = blockIdx.y == 0 ? j0 : j1;
  __shared__ float tile[kReduceRows][kMaxRank + 1];
  __shared__ float4 quarter[4][64];
  const int r = J.out.r;
  const RankOut& o = J.out;
  const int rpb = J.rpb;
  const int nblk = (J.out.rows + rpb - 1) / rpb;
  const int q4 = J.RP / 4;                    // float4 pieces per partial row
  const int lgq = __ffs(q4) - 1;
  const size_t stride4 = static_cast<size_t>(J.rows_pad) * q4;   // between splits, in float4
  const float4* part4 = reinterpret_cast<const float4*>(J.partial);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kEPT = 2;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    const int row0 = blk * rpb;
    const int nrows = J.out.rows - row0 < rpb ? J.out.rows - row0 : rpb;
    const int U = nrows * q4;
    __syncthreads();
    if (U <= 64 && J.splits > 8) {
      // Few pieces, many splits (dB: a few rows per block, a split per token
      // range): four threads per piece, each summing a quarter of the splits
      // in order, then the four quarter sums added in order.
      const int g = threadIdx.x >> 6, u = threadIdx.x & 63;
      const int rr = u >> lgq, c0 = 4 * (u & (q4 - 1));
      const bool in = u < U && c0 < r;
      const int per = (J.splits + 3) / 4;
      const int s0 = g * per, s1 = s0 + per < J.splits ? s0 + per : J.splits;
      const float4* src = part4 + static_cast<size_t>(row0 + (in ? rr : 0)) * q4 + (c0 >> 2);
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int sp0 = s0; sp0 < s1; sp0 += 8) {
        float4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = (in && sp0 + k < s1) ? __ldcg(src + static_cast<size_t>(sp0 + k) * stride4)
                                      : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          acc.x += v[k].x;
          acc.y += v[k].y;
          acc.z += v[k].z;
          acc.w += v[k].w;
        }
      }
      quarter[g][u] = acc;
      __syncthreads();
      if (g == 0 && in) {
        float4 a = quarter[0][u];
#pragma unroll
        for (int k = 1; k < 4; ++k) {
          a.x += quarter[k][u].x;
          a.y += quarter[k][u].y;
          a.z += quarter[k][u].z;
          a.w += quarter[k][u].w;
        }
        float* t = &tile[rr][c0];
        t[0] = a.x;
        t[1] = a.y;
        t[2] = a.z;
        t[3] = a.w;
      }
    }
    for (int base = 0; base < (U <= 64 && J.splits > 8 ? 0 : U); base += 256 * kEPT) {
      float4 acc[kEPT];
      const float4* src[kEPT];
      bool in[kEPT];
      int rr[kEPT], c0[kEPT];
#pragma unroll
      for (int e = 0; e < kEPT; ++e) {
        const int u = base + static_cast<int>(threadIdx.x) + 256 * e;
        rr[e] = u >> lgq;
        c0[e] = 4 * (u & (q4 - 1));
        in[e] = u < U && c0[e] < r;
        src[e] = part4 + static_cast<size_t>(row0 + (in[e] ? rr[e] : 0)) * q4 + (c0[e] >> 2);
        acc[e] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
      for (int sp0 = 0; sp0 < J.splits; sp0 += 8) {
        float4 v[kEPT][8];
#pragma unroll
        for (int e = 0; e < kEPT; ++e)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            v[e][k] = (in[e] && sp0 + k < J.splits) ? __ldcg(src[e] + static_cast<size_t>(sp0 + k) * stride4)
                                                    : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int e = 0; e < kEPT; ++e)
#pragma unroll
          for (int k = 0; k < 8; ++k) {      // split order; + 0 past the last split
            acc[e].x += v[e][k].x;
            acc[e].y += v[e][k].y;
            acc[e].z += v[e][k].z;
            acc[e].w += v[e][k].w;
          }
      }
#pragma unroll
      for (int e = 0; e < kEPT; ++e) {
        if (!in[e]) continue;
        float* t = &tile[rr[e]][c0[e]];
        t[0] = acc[e].x;
        t[1] = acc[e].y;
        t[2] = acc[e].z;
        t[3] = acc[e].w;
      }
    }
    __syncthreads();
    // row-major outputs: a warp along a row (columns across lanes)
    if ((o.f32 != nullptr && !o.transpose_f32) || o.s16 != nullptr) {
      for (int rr = warp; rr < nrows; rr += 8) {
        const size_t rowoff = static_cast<size_t>(row0 + rr) * r;
        for (int c = lane; c < r; c += 32) {
          const float v = tile[rr][c];
          if (o.f32 != nullptr && !o.transpose_f32) o.f32[rowoff + c] = v;
          if (o.s16 != nullptr) o.s16[rowoff + c] = __float2bfloat16_rn(o.scale * v);
        }
      }
    }
    // transposed outputs: a warp along a column (rows across lanes)
    if ((o.f32 != nullptr && o.transpose_f32) || o.hi != nullptr) {
      for (int c = warp; c < r; c += 8) {
        for (int rr = lane; rr < nrows; rr += 32) {
          const float v = tile[rr][c];
          const int row = row0 + rr;
          if (o.f32 != nullptr && o.transpose_f32) o.f32[static_cast<size_t>(c) * o.rows + row] = v;
          if (o.hi != nullptr) {
            const float x = o.scale * v;
            const size_t k = static_cast<size_t>(c) * o.ld + row;
            if (o.hilo_f16) {
              const __half h = __float2half_rn(x);
              static_cast<__half*>(o.hi)[k] = h;
              static_cast<__half*>(o.lo)[k] = __float2half_rn(x - __half2float(h));
            } else {
              const __nv_bfloat16 h = __float2bfloat16_rn(x);
              static_cast<__nv_bfloat16*>(o.hi)[k] = h;
              static_cast<__nv_bfloat16*>(o.lo)[k] = __float2bfloat16_rn(x - __bfloat162float(h));
            }
          }
        }
      }
    }
  }
}

// Rounding of an fp32 value to the 16-bit operand type T (bf16 or fp16).
template <typename T> __device__ __forceinline__ T to16(float v);
template <> __device__ __forceinline__ __nv_bfloat16 to16<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half to16<__half>(float v) { return __float2half_rn(v); }
__device__ __forceinline__ float from16(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float from16(__half v) { return __half2float(v); }
constexpr float kF16Max = 65504.0f;

// Backward preparation in one launch, one thread per row of the small
// operands and 8-column chunk (each thread moves one 16-byte piece of a row;
// neighbouring threads take neighbouring rows, so the transposed writes are
// coalesced): B^T ([r x d_out], bf16 or fp16) and the transposed hi/lo split
// of s*T ([r x ld]) from the forward's fp32 T (skipped when Tsave is null).
// r is a multiple of 8.
template <typename T>
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ B, int d_out, int r, T* __restrict__ Bt,
                                const float* __restrict__ Tsave, int M, float s, T* __restrict__ t_hi,
                                T* __restrict__ t_lo, int ld, uint32_t* status) {
  grid_dep_wait();
  // One thread per (row, 8-column chunk), rows fastest within a chunk so that
  // the transposed stores of neighbouring threads are contiguous.
  const long long nc = r / 8;
  const long long nb = d_out;
  const long long nt = Tsave != nullptr ? M : 0;
  bool bad = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < (nb + nt) * nc;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (i < nb * nc) {
      const int jd = static_cast<int>(i % nb), c0 = static_cast<int>(i / nb) * 8;
      const uint4 v = *reinterpret_cast<const uint4*>(B + static_cast<size_t>(jd) * r + c0);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float f = __bfloat162float(b[e]);
        Bt[static_cast<size_t>(c0 + e) * d_out + jd] = to16<T>(f);
        if (!std::is_same<T, __nv_bfloat16>::value && !(fabsf(f) <= kF16Max)) bad = true;
      }
    } else {
      const long long k = i - nb * nc;
      const int m = static_cast<int>(k % nt), c0 = static_cast<int>(k / nt) * 8;
      const float4* tp = reinterpret_cast<const float4*>(Tsave + static_cast<size_t>(m) * r + c0);
      const float4 ta = tp[0], tb = tp[1];
      const float t8[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = s * t8[e];
        const T h = to16<T>(v);
        t_hi[static_cast<size_t>(c0 + e) * ld + m] = h;
        t_lo[static_cast<size_t>(c0 + e) * ld + m] = to16<T>(v - from16(h));
        if (!std::is_same<T, __nv_bfloat16>::value && !(fabsf(v) <= kF16Max)) bad = true;
      }
    }
  }
  if (bad && status) atomicOr(status, kStatusF16Range);
}

// bf16 -> fp16 copy of a weight matrix, 8 elements per step.  bf16's 8-bit
// significand fits fp16's 11 bits, so values inside fp16's normal range
// convert exactly; |w| > 65504 flags the status word.
__global__ void convert_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, long long n,
                                   uint32_t* status) {
  grid_dep_wait();
  const long long nv = n / 8;
  bool bad = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nv;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
    __align__(16) __half h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float f = __bfloat162float(b[e]);
      h[e] = __float2half_rn(f);
      if (!(fabsf(f) <= kF16Max)) bad = true;
    }
    reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<const uint4*>(h);
  }
  if (bad && status) atomicOr(status, kStatusF16Range);
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

// Activation backward, 8 elements per thread-iteration (16-byte vectors).
//   SiLU:   dZ = dY * s(z) (1 + z (1 - s(z)))
//   SwiGLU: dZ_gate = dY * u * SiLU'(g),  dZ_up = dY * SiLU(g)
// Each dZ is emitted as fp16 hi + fp16 lo (lo = fp16(dZ - hi)): fp16's 11-bit
// significand keeps dX's rounding error well inside the tolerance, and hi + lo
// carries about 22 bits for U and dB.
template <bool kSwiglu>
__global__ void act_bwd_kernel(const __nv_bfloat16* __restrict__ dY, const float* __restrict__ Z,
                               const float* __restrict__ Zup, long long n, __half* __restrict__ g_hi,
                               __half* __restrict__ g_lo, __half* __restrict__ u_hi, __half* __restrict__ u_lo,
                               uint32_t* status) {
  grid_dep_wait();
  bool bad = false;
  const long long nv = n / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nv;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 dyv = reinterpret_cast<const uint4*>(dY)[i];
    const __nv_bfloat16* dyb = reinterpret_cast<const __nv_bfloat16*>(&dyv);
    const float4 z0 = reinterpret_cast<const float4*>(Z)[2 * i];
    const float4 z1 = reinterpret_cast<const float4*>(Z)[2 * i + 1];
    const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
    float uu[8];
    if constexpr (kSwiglu) {
      const float4 u0 = reinterpret_cast<const float4*>(Zup)[2 * i];
      const float4 u1 = reinterpret_cast<const float4*>(Zup)[2 * i + 1];
      uu[0] = u0.x; uu[1] = u0.y; uu[2] = u0.z; uu[3] = u0.w;
      uu[4] = u1.x; uu[5] = u1.y; uu[6] = u1.z; uu[7] = u1.w;
    }
    __align__(16) __half gh[8], gl[8], uh[8], ul[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float dy = __bfloat162float(dyb[e]);
      const float z = zz[e];
      const float sg = sigmoidf_(z);
      const float dsilu = sg * (1.0f + z * (1.0f - sg));
      float dg;
      if constexpr (kSwiglu) {
        dg = dy * uu[e] * dsilu;
        const float du = dy * (z * sg);
        uh[e] = __float2half_rn(du);
        ul[e] = __float2half_rn(du - __half2float(uh[e]));
        if (!(fabsf(du) <= kF16Max)) bad = true;
      } else {
        dg = dy * dsilu;
      }
      gh[e] = __float2half_rn(dg);
      gl[e] = __float2half_rn(dg - __half2float(gh[e]));
      if (!(fabsf(dg) <= kF16Max)) bad = true;
    }
    reinterpret_cast<uint4*>(g_hi)[i] = *reinterpret_cast<uint4*>(gh);
    reinterpret_cast<uint4*>(g_lo)[i] = *reinterpret_cast<uint4*>(gl);
    if constexpr (kSwiglu) {
      reinterpret_cast<uint4*>(u_hi)[i] = *reinterpret_cast<uint4*>(uh);
      reinterpret_cast<uint4*>(u_lo)[i] = *reinterpret_cast<uint4*>(ul);
    }
  }
  if (bad && status) atomicOr(status, kStatusF16Range);
}

}  // namespace lora
