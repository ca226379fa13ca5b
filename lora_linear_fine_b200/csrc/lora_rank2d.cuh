// lora_rank2d.cuh — one streaming pass over a token x feature operand Z (dZ or
// X) that feeds up to two rank-r products from the same shared-memory tile:
//
//   row product  R [tokens x r]   = Z · RB        K = features   (U  = dZ B,  RB = B^T)
//   col product  C [features x r] = Z^T · CB      K = tokens     (dB = dZ^T (sT), dA^T = X^T (sU))
//
// A 128-token x 128-feature tile of Z sits in shared memory as two
// SWIZZLE_128B boxes [feature half][128 tokens][64 features].  Read with
// K-major descriptors it is the A operand of the row product (M = tokens);
// read with MN-major descriptors (M = features, K = tokens) it is the A
// operand of the col product.  So U and dB cost one read of dZ instead of two.
//
// One CTA owns a rectangle of a_tiles token tiles x b_blocks feature blocks
// and walks it token tile by token tile (features fastest, so each token row
// is read in runs of b_blocks * 256 bytes).  Tensor memory holds one RP-column
// fp32 accumulator per token tile (row) and one 2RP-column accumulator per
// feature block (col): the hi and lo parts of the col B operand are stacked
// as one N = 2RP operand, so the Z tile is read once by the tensor core for
// both, and the epilogue adds the two halves.  The row
// B operand of the CTA's feature blocks stays resident in shared memory; the
// col B operands (hi and lo parts) of the current token tile are double
// buffered.  Partial results over the split dimension go to global memory and
// reduce_rank_kernel sums them in a fixed order; an unsplit result is written
// out directly.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 epilogue (one 32-lane TMEM quadrant each).
#pragma once

#include "lora_rank.cuh"

namespace lora {

constexpr int kRank2dThreads = 192;
constexpr int kRank2dMaxRowTiles = 32;     // row-done barriers per CTA

struct Rank2dParams {
  CUtensorMap tm_z;       // Z [mtok x F], box 64 x 128
  CUtensorMap tm_rb;      // row B [r x F], features contiguous, box 64 x RP
  CUtensorMap tm_cb[2];   // col B parts (hi, lo) [r x mtok], tokens contiguous, box 64 x RP
  int mtok, F;
  int m_tiles, f_blocks;  // 128-token tiles, 128-feature blocks
  int a_tiles, b_blocks;  // per CTA
  int fs;                 // feature splits; blockIdx.x = token_split * fs + feature_split
  float* row_partial;     // [fs][m_tiles*128][RP], or null (fs == 1: results to row_out)
  float* col_partial;     // [ts][f_blocks*128][RP], or null (one token split: results to col_out)
  RankOut row_out, col_out;
  uint32_t* status;
  // Dropout on the adapter input (col-only passes over X): keep bits [mtok x
  // mask_ld] bytes, bit j of byte b keeping feature 8 b + j; null for none.
  // The epilogue warps, idle until the end of a col-only pass, zero the
  // dropped elements of each stage's tile before the MMA warp reads it.
  const uint8_t* mask;
  int mask_ld;
};

template <int kRP, bool kRow, bool kCol>
struct Rank2dCfg {
  static constexpr int kZBox = 128 * 64 * 2;        // 16 KB
  static constexpr int kStageBytes = 2 * kZBox;     // one 128 x 128 tile
  static constexpr int kBBox = kRP * 128;           // RP rows x 64 K
  static constexpr int kRBBlock = 2 * kBBox;        // row B of one feature block (K = 128)
  static constexpr int kRBBudget = 32 * 1024;       // resident row B
  static constexpr int kMaxRB = kRow ? kRBBudget / kRBBlock : 0;
  static constexpr int kRBBytes = kRow ? kRBBudget : 0;
  static constexpr int kCBHalf = 2 * kBBox;         // hi + lo rows of one 64-token K half
  static constexpr int kCBBytes = kCol ? 2 * 2 * kCBHalf : 0;   // [buffer][K half][hi, lo]
  static constexpr int kTail = 2048;                // barriers + alignment slack
  static constexpr int kStages0 = (kSmemLimitBytes - kRBBytes - kCBBytes - kTail) / kStageBytes;
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kRBBytes + kCBBytes + kTail;
  static_assert(kStages >= 3, "ring too shallow");
  static_assert(kRBBlock % 1024 == 0 && kCBHalf % 1024 == 0, "operand alignment");
};

template <int kRP, bool kRow, bool kCol>
__global__ void __launch_bounds__(kRank2dThreads, 1) rank2d_kernel(const __grid_constant__ Rank2dParams p) {
  using C = Rank2dCfg<kRP, kRow, kCol>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_rb = smem + S * C::kStageBytes;                 // [b][2 boxes]
  uint8_t* s_cb = s_rb + C::kRBBytes;                        // [buf][K half][hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_cb + C::kCBBytes);
  uint64_t* full = bars;                                     // [S]
  uint64_t* empty = bars + S;                                // [S]
  uint64_t* rb_full = bars + 2 * S;                          // row B resident
  uint64_t* cb_full = rb_full + 1;                           // [2]
  uint64_t* cb_empty = cb_full + 2;                          // [2]
  uint64_t* col_done = cb_empty + 2;
  uint64_t* mma_done = col_done + 1;
  uint64_t* row_done = mma_done + 1;                         // [kRank2dMaxRowTiles]
  uint64_t* masked = row_done + kRank2dMaxRowTiles;          // [S] dropout: the stage's tile is masked
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(masked + S);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  AbortCtl ctl{abort_flag, p.status};
  const int tsplit = blockIdx.x / p.fs;
  const int fsplit = blockIdx.x - tsplit * p.fs;
  const int ti0 = tsplit * p.a_tiles;
  const int ti1 = ti0 + p.a_tiles < p.m_tiles ? ti0 + p.a_tiles : p.m_tiles;
  const int fj0 = fsplit * p.b_blocks;
  const int fj1 = fj0 + p.b_blocks < p.f_blocks ? fj0 + p.b_blocks : p.f_blocks;
  const int na = ti1 - ti0, nb = fj1 - fj0;     // >= 1 by the host's choice of splits
  const bool masking = kCol && !kRow && p.mask != nullptr;
  // tensor memory: row accumulators (RP columns each) first, then col accumulators (2 RP)
  const int row_cols = kRow ? na * kRP : 0;
  const uint32_t ncols_used = static_cast<uint32_t>(row_cols + (kCol ? nb * 2 * kRP : 0));
  uint32_t tcols = 32;
  while (tcols < ncols_used) tcols <<= 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(rb_full, 1);
    for (int b = 0; b < 2; ++b) { mbar_init(&cb_full[b], 1); mbar_init(&cb_empty[b], 1); }
    mbar_init(col_done, 1);
    mbar_init(mma_done, 1);
    for (int i = 0; i < kRank2dMaxRowTiles; ++i) mbar_init(&row_done[i], 1);
    for (int i = 0; i < S; ++i) mbar_init(&masked[i], 4);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, tcols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  grid_dep_wait();

  if (warp == 0) {
    if (lane == 0) {
      if constexpr (kRow) {
        mbar_arrive_expect_tx(rb_full, static_cast<uint32_t>(nb * C::kRBBlock));
        for (int j = 0; j < nb; ++j)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(s_rb + j * C::kRBBlock + h * C::kBBox, &p.tm_rb, rb_full, (fj0 + j) * 128 + h * 64, 0);
      }
      RingPos rp;
      bool ok = true;
      for (int i = 0; i < na && ok; ++i) {
        const int t0 = (ti0 + i) * 128;
        if constexpr (kCol) {
          const int buf = i & 1;
          if (!mbar_wait(&cb_empty[buf], ((i >> 1) & 1) ^ 1u, ctl)) break;
          mbar_arrive_expect_tx(&cb_full[buf], static_cast<uint32_t>(2 * C::kCBHalf));
          for (int h = 0; h < 2; ++h)
            for (int q = 0; q < 2; ++q)
              tma_load_2d(s_cb + (buf * 2 + h) * C::kCBHalf + q * C::kBBox, &p.tm_cb[q], &cb_full[buf], t0 + h * 64,
                          0);
        }
        for (int j = 0; j < nb; ++j) {
          if (!mbar_wait(&empty[rp.stage], rp.phase ^ 1u, ctl)) { ok = false; break; }
          uint8_t* st = smem + rp.stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[rp.stage], C::kStageBytes);
          const int f0 = (fj0 + j) * 128;
          tma_load_2d(st, &p.tm_z, &full[rp.stage], f0, t0);
          tma_load_2d(st + C::kZBox, &p.tm_z, &full[rp.stage], f0 + 64, t0);
          rp.next(S);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdRow = idesc_mma(128, kRP, false, false, false);
      constexpr uint32_t kIdCol = idesc_mma(128, 2 * kRP, true, false, false);
      RingPos rp;
      bool ok = true;
      if constexpr (kRow) {
        ok = mbar_wait(rb_full, 0, ctl);
        tc_fence_after();
      }
      const uint32_t srb = smem_u32(s_rb);
      const uint32_t scb = smem_u32(s_cb);
      for (int i = 0; i < na && ok; ++i) {
        const int buf = i & 1;
        if constexpr (kCol) {
          if (!mbar_wait(&cb_full[buf], (i >> 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t acc_row = tbase + static_cast<uint32_t>(i * kRP);
        for (int j = 0; j < nb; ++j) {
          if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
          if (masking && !mbar_wait(&masked[rp.stage], rp.phase, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sz = smem_u32(smem + rp.stage * C::kStageBytes);
          if constexpr (kRow) {
            // R[tile i] += Z_tile (K-major, K = 128 features) x RB[block j]
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t da = sdesc_sw128(sz + (kk >> 2) * C::kZBox + (kk & 3) * 32, 16, 1024);
              const uint64_t db = sdesc_sw128(srb + j * C::kRBBlock + (kk >> 2) * C::kBBox + (kk & 3) * 32, 16, 1024);
              mma_bf16(acc_row, da, db, kIdRow, (j == 0 && kk == 0) ? 0u : 1u);
            }
          }
          if constexpr (kCol) {
            // [C_hi | C_lo][block j] += Z_tile^T (MN-major, K = 128 tokens) x [CB_hi | CB_lo][tile i]
            const uint32_t acc_col = tbase + static_cast<uint32_t>(row_cols + j * 2 * kRP);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t da = sdesc_sw128(sz + kk * 2048, C::kZBox, 1024);
              const uint64_t db = sdesc_sw128(scb + (buf * 2 + (kk >> 2)) * C::kCBHalf + (kk & 3) * 32, 16, 1024);
              mma_bf16(acc_col, da, db, kIdCol, (i == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(&empty[rp.stage]);
          rp.next(S);
        }
        if (!ok) break;
        if constexpr (kRow) mma_commit(&row_done[i]);
        if constexpr (kCol) mma_commit(&cb_empty[buf]);
      }
      if (ok && kCol) mma_commit(col_done);
      // Teardown: every MMA issued here retires before TMEM is freed.
      mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      mbar_wait(mma_done, 0, quiet);
    }
  } else {
    // epilogue: warp w reads TMEM lanes [32 (w % 4), +32)
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float acc[kRP];
    if constexpr (kRow) {
      for (int i = 0; i < na; ++i) {
        if (!mbar_wait(&row_done[i], 0, ctl)) break;
        tc_fence_after();
        __syncwarp();
#pragma unroll
        for (int c0 = 0; c0 < kRP; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tbase + lane_off + static_cast<uint32_t>(i * kRP + c0), v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c0 + c] = __uint_as_float(v[c]);
        }
        const int tok = (ti0 + i) * 128 + lrow;
        if (p.row_partial != nullptr) {
          float* dst = p.row_partial + (static_cast<size_t>(fsplit) * p.m_tiles * 128 + tok) * kRP;
#pragma unroll
          for (int c = 0; c < kRP; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        } else if (tok < p.mtok) {
          emit_rank_row(acc, tok, p.row_out);
        }
      }
    }
    if constexpr (kCol && !kRow) {
      if (masking) {
        // Thread lrow owns token row lrow of both [128 x 64] SWIZZLE_128B boxes
        // of every stage and the row's 16 keep bytes for the stage's 128
        // features, loaded one stage ahead so that their latency hides behind
        // the wait for the tiles.
        const bool vec = (reinterpret_cast<uintptr_t>(p.mask) % 16) == 0 && p.mask_ld % 16 == 0;
        auto keep = [&](int i, int j, uint32_t (&m)[4]) {
          const int tok = (ti0 + i) * 128 + lrow;
          const bool in_rows = tok < p.mtok;
          const uint8_t* mrow = p.mask + static_cast<size_t>(in_rows ? tok : 0) * p.mask_ld;
          load_keep_bytes<16>(mrow, (fj0 + j) * 16, p.mask_ld, in_rows, vec, m);
        };
        uint32_t cur[4], nxt[4];
        keep(0, 0, cur);
        RingPos rp;
        bool ok = true;
        for (int i = 0; i < na && ok; ++i) {
          for (int j = 0; j < nb; ++j) {
            const bool last_j = j + 1 == nb;
            if (!last_j || i + 1 < na) keep(last_j ? i + 1 : i, last_j ? 0 : j + 1, nxt);
            if (!mbar_wait(&full[rp.stage], rp.phase, ctl)) { ok = false; break; }
            uint8_t* st = smem + rp.stage * C::kStageBytes;
            mask_sw128_rows<2>(st + lrow * 128, C::kZBox, lrow, cur);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&masked[rp.stage]);
#pragma unroll
            for (int w = 0; w < 4; ++w) cur[w] = nxt[w];
            rp.next(S);
          }
        }
      }
    }
    if constexpr (kCol) {
      if (mbar_wait(col_done, 0, ctl)) {
        tc_fence_after();
        __syncwarp();
        for (int j = 0; j < nb; ++j) {
          const uint32_t col_base = tbase + lane_off + static_cast<uint32_t>(row_cols + j * 2 * kRP);
#pragma unroll
          for (int c0 = 0; c0 < kRP; c0 += 16) {
            uint32_t vh[16], vl[16];
            tmem_ld16(col_base + c0, vh);
            tmem_ld16(col_base + kRP + c0, vl);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c0 + c] = __uint_as_float(vh[c]) + __uint_as_float(vl[c]);
          }
          const int feat = (fj0 + j) * 128 + lrow;
          if (p.col_partial != nullptr) {
            float* dst = p.col_partial + (static_cast<size_t>(tsplit) * p.f_blocks * 128 + feat) * kRP;
#pragma unroll
            for (int c = 0; c < kRP; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
          } else if (feat < p.F) {
            emit_rank_row(acc, feat, p.col_out);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }
}

// Feature blocks whose row B fits the resident budget.
constexpr int rank2d_max_rb(int RP) { return (32 * 1024) / (2 * RP * 128); }

// Split of an (m_tiles x f_blocks) tile grid into rectangles for rank2d_kernel.
struct Rank2dSplit {
  int a = 0, b = 0, ts = 0, fs = 0;
};

// Choose a x b rectangles: tensor memory ((a + 2b) RP columns, or the used
// product's), the resident row B (b blocks), at most kRank2dMaxRowTiles row
// tiles; among those, the least estimated time: the bytes a CTA of the most
// loaded wave brings in (its Z tiles, with runs per token row shorter than
// 2 KB charged for their lower DRAM efficiency; the col B operand once per
// token tile; the resident row B once), times the CTAs of that wave, plus the
// partials written and read back.  The col B operand (hi and lo, 512 RP bytes
// per token tile) is as large as a Z tile at RP = 64, so a CTA that walks one
// feature block per token tile spends half its loads on it.
inline Rank2dSplit rank2d_split(int m_tiles, int f_blocks, int RP, bool row, bool col, int max_rb, int ctas) {
  Rank2dSplit best;
  double best_cost = 0.0;
  const int tcols = 512 / RP;                 // RP-column units of tensor memory
  int bmax = f_blocks;
  if (row && max_rb < bmax) bmax = max_rb;
  if (col && !row && tcols / 2 < bmax) bmax = tcols / 2;
  if (row && col && (tcols - 1) / 2 < bmax) bmax = (tcols - 1) / 2;
  for (int b = 1; b <= bmax; ++b) {
    const int fs = (f_blocks + b - 1) / b;
    const int be = (f_blocks + fs - 1) / fs;
    int a_max = kRank2dMaxRowTiles;
    if (row && col) a_max = tcols - 2 * be < a_max ? tcols - 2 * be : a_max;
    else if (row) a_max = tcols < a_max ? tcols : a_max;
    else a_max = m_tiles;                      // col only: token tiles cost no tensor memory
    if (a_max < 1) continue;
    int ts = ctas / fs;
    if (ts < 1) ts = 1;
    if (ts > m_tiles) ts = m_tiles;
    int a = (m_tiles + ts - 1) / ts;
    if (a > a_max) a = a_max;
    ts = (m_tiles + a - 1) / a;
    const long long n = static_cast<long long>(ts) * fs;
    const long long waves = (n + ctas - 1) / ctas;
    const double tile = 32768.0;
    const double width = static_cast<double>(waves) * static_cast<double>(n < ctas ? n : ctas);
    double cost = width * a * be * tile;
    const double run = be * 256.0;
    if (run < 2048.0) cost *= 1.0 + 0.5 * (1.0 - run / 2048.0);
    if (col) cost += width * a * 512.0 * RP;          // col B (hi + lo) per token tile
    if (row) cost += width * be * 256.0 * RP;         // resident row B
    if (row && fs > 1) cost += 2.0 * fs * m_tiles * 128.0 * RP * 4.0;
    if (col && ts > 1) cost += 2.0 * ts * f_blocks * 128.0 * RP * 4.0;
    if (best.a == 0 || cost < best_cost) {
      best_cost = cost;
      best.a = a;
      best.b = be;
      best.ts = ts;
      best.fs = fs;
    }
  }
  return best;
}

}  // namespace lora
