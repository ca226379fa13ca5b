// lora_mma.cuh — the fused LoRA-adapted linear layer as one tcgen05 GEMM whose
// K-loop carries the LoRA branch as extra K-blocks:
//
//   forward   Z  = X W^T + s T B^T  = [ X | sT ] [ W | B ]^T      (T = X A^T)
//   backward  dX = dZ W  + s U A    = [ dZ | sU ] [ W ; A ]       (U = dZ B)
//
// T (U) comes from the rank pass (lora_rank.cuh), which also writes s*T as bf16
// [M x r]; the GEMM's last K-blocks per tile (one per 64 of r and projection)
// multiply that tile of s*T (K = r, zero-filled by TMA up to a whole 64-wide
// block) with the matching rows of B (A).
// The up-projection thus runs on the tensor cores inside the same accumulator,
// with no hand-off between the epilogue and the MMA issuer, which leaves the
// tensor memory free for a double-buffered accumulator: 2 x 256 fp32 columns.
// The backward reads W and A either in place as MN-major operands (b_mn = 1),
// or as K-major copies W^T and A^T that it writes first (b_mn = 0): the copy
// costs one read and one write of W, and the tensor pipe then runs as in the
// forward, where the MN-major read left it idle ~10 % more often on q_proj.
// The epilogue of tile i (drain, activation, bf16 store) overlaps the K-loop of
// tile i + 1.
//
// kPair = false: one CTA per 128 x 256 tile (tcgen05 cta_group::1).
// kPair = true : a cluster of two CTAs per 256 x 256 tile (cta_group::2): CTA c
//   holds rows [128c, 128c + 128) of the M-side operand and half of the N-side
//   operand; the leader (c = 0) issues the MMAs; each CTA's tensor memory holds
//   its own 128 accumulator rows.  The TMA transactions of both CTAs complete on
//   the leader's `full` barrier; the leader's commits arrive on both CTAs'
//   barriers; both CTAs' epilogues arrive on the leader's `acc_empty` barriers.
//
// SwiGLU forward: the N-side operand of a tile is 128 gate rows + 128 up rows
// of the same outputs (paired kernel: gate in CTA 0, up in CTA 1); the LoRA
// blocks are two N = 128 products, one per projection.  SwiGLU backward: the
// K-loop runs through both projections (dZ_gate W_gate + dZ_up W_up + LoRA).
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..9 epilogue (two warps per 32-lane TMEM quadrant).
#pragma once

#include "sm100.cuh"
#include "lora_norm_rope.cuh"

namespace lora {

constexpr int kMmaThreads = 320;

// kEpi values
// kMEpiRope: identity, then the rotary embedding of each token's heads on the
// fp32 accumulator (lora_norm_rope.cuh) before the bf16 store.
// kMEpiCeFwd: the output projection's logits z = H W^T of a 256 x 256 tile are
// reduced in the epilogue to one (max, sum of exp(z - max)) pair per token and
// 128-column block, and the label's logit is picked up; no logit is stored.
// kMEpiCeGrad: the same logits recomputed and turned into the cross-entropy
// gradient (exp(z - lse) - onehot(label)) * scale, stored as bf16.
// kMEpiGradF32 / kMEpiGradF16F32: the dX GEMM (bf16 / fp16 operands) writing
// or adding to an fp32 dX, staged through shared memory so that each global
// access covers whole sectors of one row.
// kMEpiGradDrop / kMEpiGradF16Drop: the dX GEMM (bf16 / fp16 operands) of a
// layer with dropout on the adapter input; its LoRA K-blocks go first, the
// epilogue warps zero the dropped entries of that term in tensor memory, and
// the main K-blocks accumulate on top before the one bf16 rounding.
// kMEpiIdentityT / kMEpiRopeT: the forward of one projection (identity, or
// rotated as kMEpiRope) with T = X A^T accumulated inside the GEMM by the T
// tiles (MmaParams: tm_am, t_shared).
// kMEpiCeFwdZ: kMEpiCeFwd that also stores the fp32 logits.
enum MmaEpi : int {
  kMEpiIdentity = 0, kMEpiSilu = 1, kMEpiSwiglu = 2, kMEpiGrad = 3, kMEpiGradF16 = 4, kMEpiRope = 5,
  kMEpiCeFwd = 6, kMEpiCeGrad = 7, kMEpiGradF32 = 8, kMEpiGradF16F32 = 9, kMEpiGradDrop = 10,
  kMEpiGradF16Drop = 11, kMEpiIdentityT = 12, kMEpiCeFwdZ = 13, kMEpiRopeT = 14
};

// Dropout on the adapter input, dX epilogue (kMEpiGradDrop / kMEpiGradF16Drop).
// Dropout keep bits of the dX GEMM's outputs (the elements of X): [M x N/8]
// bytes, bit j of byte b (least significant first) keeping column 8 b + j.
struct DropEpi {
  const uint8_t* mask;
};

// Output projection fused with the cross-entropy loss (rows = tokens of this
// launch, columns = vocabulary entries).
struct CeParams {
  const int32_t* labels;  // [M] label per token; < 0 ignored (also >= N: flagged by the combine kernel)
  float2* part;           // kMEpiCeFwd: [2 * n_tiles][M] (max, sum exp(z - max)) per 128-column block
  float* zlab;            // kMEpiCeFwd: [M] z[label] (written by the block holding the label)
  const float* lse;       // kMEpiCeGrad: [M] log-sum-exp of each token's logits
  const float* scale;     // kMEpiCeGrad: device scalar, d(loss) / (number of valid tokens)
};

struct MmaParams {
  CUtensorMap tm_a[2];    // M-side operand per pair      fwd: X            bwd: dZ_j
  CUtensorMap tm_w[2];    // N-side operand per pair      fwd: W_j          bwd: W_j (b_mn) or W_j^T
  CUtensorMap tm_la[2];   // LoRA block, M side           s*T_j / s*U_j   bf16 [M x r]
  CUtensorMap tm_lb[2];   // LoRA block, N side           fwd: B_j [d_out x r]   bwd: A_j (b_mn) or A_j^T
  int M, N, K;            // output rows / columns (per projection for SwiGLU fwd) / reduction per pair
  int lora_ksteps;        // 16-wide K steps of a projection's LoRA blocks: ceil(r / 16) <= 8; 0 = none
  __nv_bfloat16* out;     // [M x N]
  float* z_save;          // [npair][M x N] fp32 or null (SiLU / SwiGLU forward)
  uint32_t* status;
  int m_tiles, n_tiles, num_tiles;
  int group;              // raster group width (tiles)
  int group_along_n;      // 0: groups of `group` M tiles sweep all N tiles (the N-side operand stays in L2)
                          // 1: groups of `group` N tiles sweep all M tiles (the M-side operand stays in L2)
  int b_mn;               // backward: N-side operands read MN-major (W [K x N], A [r x N]) instead of K-major copies
  RopeTables rope;        // kMEpiRope: positions and cos / sin tables (half = 32 or 64)
  float* out_f32;         // backward: fp32 dX [M x N] instead of the bf16 `out` (null: bf16)
  int out_acc;            // with out_f32: dX += the product (else dX = the product)
  CeParams ce;            // kMEpiCeFwd / kMEpiCeGrad
  DropEpi drop;           // kMEpiGradDrop / kMEpiGradF16Drop
  // kMEpiIdentityT (forward): T = X A^T accumulates in the second accumulator
  // buffer during the main K-loop of a T tile.  t_shared = 0: every tile is
  // a T tile (one tile per unit).  t_shared = 1: the first m_tiles tiles are
  // the N-tile-0 tiles of each row block, one per unit and each its unit's
  // first tile; they publish bf16(s T) to st_out, and the row block's other
  // tiles load it from there (tm_la[0]) for their LoRA block once the
  // publishing CTA's flag bits are set.
  CUtensorMap tm_am;      // A [r x K], box 64 x am_rows (this CTA's am_rows rows of the padded rank)
  CUtensorMap tm_out;     // set by the launcher for the TMA-store epilogues: bf16 out [M x N], box 64 x 32;
                          // kMEpiCeFwdZ, kMEpiGradF32, kMEpiGradF16F32: fp32 out_f32 [M x N], box 32 x 32;
                          // kMEpiRope: bf16 out [M x N], box 32 x 32, 64-byte swizzle
  CUtensorMap tm_z[2];    // SiLU / SwiGLU forward with z_save: fp32 Z (SwiGLU: gate, up) [M x N], box 32 x 32
  int am_rows;            // rows of A per CTA: RP / (CTAs per unit)
  int rp;                 // the rank padded to a multiple of 16 (the T MMA's N)
  int r;                  // the rank
  float lora_scale;       // s: the LoRA block's operand is bf16(s T)
  float* t_save;          // fp32 T [M x r] for the backward (written by the N-tile-0 units), or null
  int t_shared;
  __nv_bfloat16* st_out;  // t_shared: bf16(s T) [M x r], row-major
  uint32_t* t_flags;      // t_shared: [0] exit count, [1..kTFlagWords] flag bits; zero at rest
};

// Flag words of the shared-T forward: 4 bits (one per writing epilogue warp)
// per CTA of each T tile; the last CTA to exit zeroes them again.
constexpr int kTFlagWords = 19;

template <bool kPair, bool kBwd, int kNPair, int kEpi>
struct MmaCfg {
  static constexpr bool kSwigluFwd = (!kBwd) && (kEpi == kMEpiSwiglu);
  static constexpr int kCtas = kPair ? 2 : 1;
  static constexpr int kTileM = 128 * kCtas;                 // rows per (pair) tile
  static constexpr int kOutCols = kSwigluFwd ? 128 : 256;    // output columns per tile
  static constexpr int kKPairs = kBwd ? kNPair : 1;          // projections walked along K
  static constexpr int kLoraProj = kNPair;                   // projections with a LoRA branch per tile
  static constexpr int kABytes = 128 * 64 * 2;               // 16 KB
  static constexpr int kBRows = 256 / kCtas;                 // N-side rows held per CTA
  static constexpr int kBBytes = kBRows * 64 * 2;            // 32 KB (single) / 16 KB (pair)
  // kMEpiIdentityT: rows of A (the rank, up to 64 in all) per stage and CTA,
  // in a ring of their own after the main stages, which keep the plain
  // kernel's layout
  static constexpr bool kTFused = kEpi == kMEpiIdentityT || kEpi == kMEpiRopeT;
  static constexpr int kAMBytes = kTFused ? (64 / kCtas) * 64 * 2 : 0;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // Epilogues that store fp32 Z (SiLU, SwiGLU) stage each warp's rows through
  // shared memory (4 KB per warp) so that global stores are row-contiguous.
  static constexpr bool kStaged = kSwigluFwd || kEpi == kMEpiSilu || kEpi == kMEpiGradF32 || kEpi == kMEpiGradF16F32;
  // Dropout on the adapter input (backward, one projection): the masked
  // LoRA term is formed in the accumulator before the main K-loop.
  static constexpr bool kDropEpi = kEpi == kMEpiGradDrop || kEpi == kMEpiGradF16Drop;
  // The bf16 epilogues without their own output path (identity forward,
  // dX) stage each warp's rows in shared memory as well and write them with
  // TMA stores: per-thread 16-byte stores scattered over 32 rows slowed the
  // loads that feed the tensor core by 1.3-1.8k cycles per tile.
  static constexpr bool kTmaOut = !(kSwigluFwd || kEpi == kMEpiSilu || kEpi == kMEpiRope || kEpi == kMEpiRopeT ||
                                    kEpi == kMEpiGradF32 ||
                                    kEpi == kMEpiGradF16F32 || kEpi == kMEpiCeFwd || kEpi == kMEpiCeFwdZ ||
                                    kEpi == kMEpiCeGrad);
  // The fp32 logits of kMEpiCeFwdZ and the fp32 dX of kMEpiGradF32 /
  // kMEpiGradF16F32 (stored, or added at L2 with out_acc) leave the same way.
  static constexpr bool kTmaZ = kEpi == kMEpiCeFwdZ || kEpi == kMEpiGradF32 || kEpi == kMEpiGradF16F32;
  // ... and the rotated bf16 output of kMEpiRope, in 32-column boxes.
  static constexpr bool kTmaRope = kEpi == kMEpiRope || kEpi == kMEpiRopeT;
  // ... and the SiLU / SwiGLU forward's bf16 Y and fp32 Z.
  static constexpr bool kTmaAct = kSwigluFwd || (kEpi == kMEpiSilu && !kBwd);
  static constexpr int kEpiStageBytes = (kStaged || kTmaOut || kTmaZ || kTmaRope) ? 8 * 4096 : 0;
  static constexpr int kStages0 = (kSmemLimitBytes - 2048 - kEpiStageBytes) / (kStageBytes + kAMBytes);
  static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
  static constexpr int kAMOff = kStages * kStageBytes;              // the A-rows ring
  static constexpr int kRingBytes = kStages * (kStageBytes + kAMBytes);
  static constexpr int kSmemBytes = kRingBytes + kEpiStageBytes + 2048;
  static constexpr uint32_t kTmemCols = 512;                 // 2 accumulator buffers
  static_assert(kStages >= 3, "ring too shallow");
};

// Tile t of the raster.  Consecutive tiles (processed at the same time by
// neighbouring CTAs) share their N-side operand (group_along_n = 0: M fastest
// inside a group of `group` M tiles) or their M-side operand (group_along_n = 1:
// M fastest inside a group of `group` N tiles, so the whole M-side operand is
// swept per group and stays in L2 while the N-side operand streams once).
// With a shared T (t_shared), tiles 0 .. m_tiles - 1 are the N-tile-0 tiles
// in row order, and the raster covers the remaining N tiles.
__device__ __forceinline__ void mma_tile_coords(int t, const MmaParams& p, int& mt, int& nt) {
  int n_tiles = p.n_tiles, nt0 = 0;
  if (p.t_shared) {
    if (t < p.m_tiles) { mt = t; nt = 0; return; }
    t -= p.m_tiles;
    n_tiles -= 1;
    nt0 = 1;
  }
  if (p.group_along_n) {
    const int per_group = p.group * p.m_tiles;
    const int g = t / per_group;
    const int idx = t - g * per_group;
    mt = idx % p.m_tiles;
    nt = nt0 + g * p.group + idx / p.m_tiles;
  } else {
    const int per_group = p.group * n_tiles;
    const int g = t / per_group;
    const int first_m = g * p.group;
    const int rem = p.m_tiles - first_m;
    const int gm = rem < p.group ? rem : p.group;
    const int idx = t - g * per_group;
    mt = first_m + idx % gm;
    nt = nt0 + idx / gm;
  }
}

template <bool kPair>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const AbortCtl& ctl) {
  if constexpr (kPair) return mbar_wait_cluster(bar, parity, ctl);
  else return mbar_wait(bar, parity, ctl);
}

template <bool kPair, bool kBwd, int kNPair, int kEpi>
__global__ void __launch_bounds__(kMmaThreads, 1) lora_mma_kernel(const __grid_constant__ MmaParams p) {
  using C = MmaCfg<kPair, kBwd, kNPair, kEpi>;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_stage = smem + C::kRingBytes;               // [8 warps][4 KB] (kStaged)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kRingBytes + C::kEpiStageBytes);
  uint64_t* full = bars;                  // [S]
  uint64_t* empty = bars + S;             // [S]
  uint64_t* acc_full = bars + 2 * S;      // [2] accumulator buffer b complete
  uint64_t* acc_empty = acc_full + 2;     // [2] accumulator buffer b drained
  uint64_t* mma_done = acc_full + 4;
  uint64_t* lora_done = acc_full + 5;     // [2] dropout: the LoRA term of buffer b is in the accumulator
  uint64_t* masked = acc_full + 7;        // [2] dropout: its dropped entries are zeroed
  uint64_t* t_done = acc_full + 9;        // fused T: the main K-loop (and T) is complete
  uint64_t* t_ready = acc_full + 10;      // fused T: bf16(s T) is in the LoRA stage's A area
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 11);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = kPair ? cluster_ctarank() : 0u;
  const bool leader = crank == 0;
  const int unit = kPair ? (blockIdx.x >> 1) : blockIdx.x;        // scheduling unit (CTA or pair)
  const int nunits = kPair ? (gridDim.x >> 1) : gridDim.x;
  AbortCtl ctl{abort_flag, p.status};
  if constexpr (C::kTFused) {
    // The fused T needs its T tiles to be their units' first tiles (one tile
    // per unit, or with a shared T one row block per unit); anything else is
    // refused before any barrier, tensor memory or cluster step.
    const bool bad_sched = p.t_shared ? (p.m_tiles > nunits || p.st_out == nullptr || p.t_flags == nullptr ||
                                         p.m_tiles * C::kCtas * 4 > 32 * kTFlagWords)
                                      : p.num_tiles > nunits;
    if (bad_sched || p.rp < 16 || p.rp > 64 || p.rp % 16 != 0 || p.am_rows * C::kCtas != p.rp) {
      if (threadIdx.x == 0 && p.status != nullptr) atomicOr(p.status, kStatusBadArgument);
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    // acc_empty: one arrival per epilogue warp of every CTA of the unit
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 8 * C::kCtas); }
    for (int b = 0; b < 2; ++b) { mbar_init(&lora_done[b], 1); mbar_init(&masked[b], 8 * C::kCtas); }
    mbar_init(t_done, 1);
    mbar_init(t_ready, 4 * C::kCtas);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < (C::kSwigluFwd ? 1 : kNPair); ++j) tma_prefetch_desc(&p.tm_a[j]);
    for (int j = 0; j < kNPair; ++j) tma_prefetch_desc(&p.tm_w[j]);
    if (p.lora_ksteps > 0)
      for (int j = 0; j < kNPair; ++j) { tma_prefetch_desc(&p.tm_la[j]); tma_prefetch_desc(&p.tm_lb[j]); }
  }
  if (warp == 1) {
    if constexpr (kPair) { tmem_alloc_pair(tmem_slot, C::kTmemCols); tmem_relinquish_pair(); }
    else { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  grid_dep_wait();
  const int nkb = (p.K + 63) / 64;
  const int lkb = (p.lora_ksteps + 3) / 4;                   // 64-wide LoRA K-blocks per projection
  const int nlora = C::kLoraProj * lkb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      RingPos rp;
      uint32_t issued = 0;
      bool ok = true;
      // One TMA box into this CTA's shared memory; completion on the stage's
      // `full` barrier (the leader's for a pair).
      auto load = [&](void* dst, const CUtensorMap* tm, uint32_t stage, int x, int y, uint64_t pol) {
        if constexpr (kPair) tma_load_2d_pair(dst, tm, mapa_shared(smem_u32(&full[stage]), 0), x, y, pol);
        else tma_load_2d_hint(dst, tm, &full[stage], x, y, pol);
      };
      // Bytes one stage brings into ALL CTAs of the unit: main and backward
      // LoRA blocks fill both areas; a forward SwiGLU LoRA block fills the A
      // area and 128 rows of N-side operand (64 per CTA of a pair).
      constexpr uint32_t kTxFull = C::kCtas * C::kStageBytes;
      constexpr uint32_t kTxSwigluLora = C::kCtas * C::kABytes + 128 * 64 * 2;
      // This CTA's first row and the tile's first column of tile t.
      auto origin = [&](int t, int& m0, int& n0) {
        int mt, nt;
        mma_tile_coords(t, p, mt, nt);
        m0 = mt * C::kTileM + 128 * static_cast<int>(crank);
        n0 = nt * C::kOutCols;
      };
      // The blocks of the tile at (m0, n0), each into the next ring stage:
      // the main K-blocks (projection j, columns [k0, k0 + 64) of K), then
      // the LoRA blocks; false if the wait for the stage gave up.  Main and
      // LoRA blocks go through separate functions that the tile loops call
      // in order, so that the per-block path (which sets the pace of the
      // whole pipeline) carries no branch or division between the two kinds.
      auto put_main = [&](int m0, int n0, int j, int k0) -> bool {
        if (!wait_bar<kPair>(&empty[rp.stage], rp.phase ^ 1u, ctl)) return false;
        uint8_t* sa = smem + rp.stage * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        const uint32_t fb = rp.stage;
        if (leader) mbar_arrive_expect_tx(&full[rp.stage], kTxFull);
        {
          load(sa, &p.tm_a[j], fb, k0, m0, pol_stream);
          if constexpr (!kBwd) {
            if constexpr (C::kSwigluFwd) {
              if constexpr (kPair) load(sb, &p.tm_w[crank], fb, k0, n0, pol_keep);
              else {
                load(sb, &p.tm_w[0], fb, k0, n0, pol_keep);
                load(sb + C::kBBytes / 2, &p.tm_w[1], fb, k0, n0, pol_keep);
              }
            } else {
              load(sb, &p.tm_w[0], fb, k0, n0 + C::kBRows * static_cast<int>(crank), pol_keep);
            }
          } else if (p.b_mn) {
#pragma unroll
            for (int b = 0; b < C::kBRows / 64; ++b)
              load(sb + b * 8192, &p.tm_w[j], fb, n0 + C::kBRows * static_cast<int>(crank) + 64 * b, k0, pol_keep);
          } else {
            // a K-major N-side operand (rows = outputs of dX); the library's
            // backward launches read W in place (b_mn) instead
            load(sb, &p.tm_w[j], fb, k0, n0 + C::kBRows * static_cast<int>(crank), pol_keep);
          }
        }
        ++issued;
        rp.next(S);
        return true;
      };
      auto put_lora = [&](int m0, int n0, int lb) -> bool {
        if (!wait_bar<kPair>(&empty[rp.stage], rp.phase ^ 1u, ctl)) return false;
        uint8_t* sa = smem + rp.stage * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        const uint32_t fb = rp.stage;
        if (leader) mbar_arrive_expect_tx(&full[rp.stage], C::kSwigluFwd ? kTxSwigluLora : kTxFull);
        {
          // LoRA block lb, of projection j: s*T_j (s*U_j) rows and B_j (A_j)
          // rows, K = r columns [kx, kx + 64) of the rank, zero-filled past r
          const int j = lb / lkb;
          const int kx = (lb - j * lkb) * 64;
          load(sa, &p.tm_la[j], fb, kx, m0, pol_keep);
          if constexpr (!kBwd) {
            if constexpr (C::kSwigluFwd) {
              // N = 128 outputs of projection j: 128 rows (single) or 64 per CTA (pair)
              load(sb, &p.tm_lb[j], fb, kx, n0 + 64 * static_cast<int>(crank), pol_keep);
            } else {
              load(sb, &p.tm_lb[0], fb, kx, n0 + C::kBRows * static_cast<int>(crank), pol_keep);
            }
          } else if (p.b_mn) {
#pragma unroll
            for (int b = 0; b < C::kBRows / 64; ++b)
              load(sb + b * 8192, &p.tm_lb[j], fb, n0 + C::kBRows * static_cast<int>(crank) + 64 * b, kx, pol_keep);
          } else {
            load(sb, &p.tm_lb[j], fb, kx, n0 + C::kBRows * static_cast<int>(crank), pol_keep);   // A^T rows
          }
        }
        ++issued;
        rp.next(S);
        return true;
      };
      // Fused T, a T tile's block blk (one identity projection): a main block
      // brings X, W and this CTA's am_rows rows of A (into the A-rows ring);
      // the LoRA block brings only B, since the epilogue warps write bf16(s T)
      // into its A area.  Kept apart from put so that the other tiles run the
      // plain per-block path: the producer's per-block work sets the pace of
      // the whole pipeline.
      auto put_t = [&](int m0, int n0, int blk) -> bool {
        if (!wait_bar<kPair>(&empty[rp.stage], rp.phase ^ 1u, ctl)) return false;
        uint8_t* sa = smem + rp.stage * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        const uint32_t fb = rp.stage;
        if (blk < nkb) {
          if (leader)
            mbar_arrive_expect_tx(&full[rp.stage],
                                  C::kCtas * (C::kABytes + C::kBBytes + static_cast<uint32_t>(p.am_rows) * 128u));
          load(sa, &p.tm_a[0], fb, blk * 64, m0, pol_stream);
          load(smem + C::kAMOff + rp.stage * C::kAMBytes, &p.tm_am, fb, blk * 64,
               p.am_rows * static_cast<int>(crank), pol_keep);
          load(sb, &p.tm_w[0], fb, blk * 64, n0 + C::kBRows * static_cast<int>(crank), pol_keep);
        } else {
          if (leader) mbar_arrive_expect_tx(&full[rp.stage], C::kCtas * C::kBBytes);
          load(sb, &p.tm_lb[0], fb, (blk - nkb) * 64, n0 + C::kBRows * static_cast<int>(crank), pol_keep);
        }
        ++issued;
        rp.next(S);
        return true;
      };
      const int nmain = C::kKPairs * nkb;
      if constexpr (C::kDropEpi) {
        // Dropout: the tensor core first writes the LoRA term of a tile into
        // its accumulator, the epilogue warps zero its dropped entries, then
        // the main K-blocks accumulate on top.  The next tile's LoRA blocks
        // ride in the middle of this tile's main blocks, so that the masking
        // of the other accumulator buffer overlaps this tile's K-loop:
        //   L(t0), main(t0)[0, h), L(t1), main(t0)[h, n), main(t1)[0, h), L(t2), ...
        const int h = nmain / 2;
        int m0, n0, m1 = 0, n1 = 0;
        for (int t = unit; t < p.num_tiles && ok; t += nunits) {
          origin(t, m0, n0);
          if (t == unit)
            for (int lb = 0; lb < nlora && ok; ++lb) ok = put_lora(m0, n0, lb);
          for (int blk = 0; blk < h && ok; ++blk) ok = put_main(m0, n0, 0, blk * 64);
          if (t + nunits < p.num_tiles) {
            origin(t + nunits, m1, n1);
            for (int lb = 0; lb < nlora && ok; ++lb) ok = put_lora(m1, n1, lb);
          }
          for (int blk = h; blk < nmain && ok; ++blk) ok = put_main(m0, n0, 0, blk * 64);
        }
      } else {
        int m0, n0;
        for (int t = unit; t < p.num_tiles && ok; t += nunits) {
          origin(t, m0, n0);
          if constexpr (C::kTFused) {
            if (!p.t_shared || t < p.m_tiles) {
              for (int blk = 0; blk < nmain + nlora && ok; ++blk) ok = put_t(m0, n0, blk);
            } else {
              // the row block's T tile publishes bf16(s T): wait for this
              // CTA's four flag bits before the LoRA block loads it
              for (int kb = 0; kb < nkb && ok; ++kb) ok = put_main(m0, n0, 0, kb * 64);
              const int bit = ((m0 - 128 * static_cast<int>(crank)) / C::kTileM * C::kCtas + static_cast<int>(crank)) * 4;
              if (ok) ok = flag_wait_all(p.t_flags + 1 + bit / 32, 0xFu << (bit % 32), ctl);
              fence_proxy_async_global();
              for (int lb = 0; lb < nlora && ok; ++lb) ok = put_lora(m0, n0, lb);
            }
          } else {
            for (int j = 0; j < C::kKPairs && ok; ++j)
              for (int kb = 0; kb < nkb && ok; ++kb) ok = put_main(m0, n0, j, kb * 64);
            for (int lb = 0; lb < nlora && ok; ++lb) ok = put_lora(m0, n0, lb);
          }
        }
      }
      if (!ok && leader) {
        RingPos q = rp;
        volatile uint32_t zero = 0u;
        AbortCtl quiet{&zero, nullptr};
        for (uint32_t i = 0; i < (issued < (uint32_t)S ? issued : (uint32_t)S); ++i) {
          if (q.stage == 0) { q.stage = S - 1; q.phase ^= 1u; } else { --q.stage; }
          wait_bar<kPair>(&full[q.stage], q.phase, quiet);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      constexpr bool kF16 = (kEpi == kMEpiGradF16 || kEpi == kMEpiGradF16F32 || kEpi == kMEpiGradF16Drop);
      constexpr int kM = C::kTileM;
      // N-side operand MN-major only in a backward that reads W and A in place
      const bool bmn = kBwd && p.b_mn != 0;
      const uint32_t kIdMain = bmn ? idesc_mma(kM, 256, false, true, kF16) : idesc_mma(kM, 256, false, false, kF16);
      // LoRA block: bf16 s*T/s*U against bf16 B (fwd) / A or A^T (bwd)
      const uint32_t kIdLora = bmn ? idesc_mma(kM, 256, false, true, false)
                                   : idesc_mma(kM, C::kSwigluFwd ? 128 : 256, false, false, false);
      constexpr uint16_t kBoth = 0x3;
      auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (kPair) mma_bf16_pair(d, a, b, id, acc);
        else mma_bf16(d, a, b, id, acc);
      };
      auto commit = [&](uint64_t* bar) {
        if constexpr (kPair) mma_commit_pair(bar, kBoth);
        else mma_commit(bar);
      };
      const uint32_t kIdT = idesc_mma(kM, C::kTFused ? p.rp : 16, false, false, false);
      RingPos rp;
      const int nmain = C::kKPairs * nkb;
      // Block blk of a tile (main K-blocks first, then the LoRA blocks) from
      // the next ring stage into the accumulator at dacc.  The first MMA of a
      // tile starts the accumulator: main block 0 normally, LoRA block 0 with
      // dropout (where the main blocks then accumulate on the masked term).
      auto take = [&](int blk, uint32_t dacc) -> bool {
        if (!wait_bar<kPair>(&full[rp.stage], rp.phase, ctl)) return false;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
        if (blk < nmain) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = bmn ? sdesc_sw128(sb + kk * 2048, 8192, 1024) : sdesc_sw128(sb + kk * 32, 16, 1024);
            mma(dacc, da, db, kIdMain, (!C::kDropEpi && blk == 0 && kk == 0) ? 0u : 1u);
          }
        } else {
          const int lb = blk - nmain;
          const int j = lb / lkb;
          const int steps = p.lora_ksteps - 4 * (lb - j * lkb);     // this block's 16-wide steps
          const uint32_t dcol = C::kSwigluFwd ? static_cast<uint32_t>(128 * j) : 0u;
          for (int kk = 0; kk < (steps < 4 ? steps : 4); ++kk) {
            const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = bmn ? sdesc_sw128(sb + kk * 2048, 8192, 1024) : sdesc_sw128(sb + kk * 32, 16, 1024);
            mma(dacc + dcol, da, db, kIdLora, (C::kDropEpi && lb == 0 && kk == 0) ? 0u : 1u);
          }
        }
        commit(&empty[rp.stage]);
        rp.next(S);
        return true;
      };
      // Fused T, a T tile's main block blk: the main product and T += X tile
      // x (rows of A)^T into the second buffer's columns.
      auto take_t = [&](int blk, uint32_t dacc) -> bool {
        if (!wait_bar<kPair>(&full[rp.stage], rp.phase, ctl)) return false;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + rp.stage * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
        const uint32_t sam = smem_u32(smem + C::kAMOff + rp.stage * C::kAMBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = sdesc_sw128(sa + kk * 32, 16, 1024);
          const uint32_t acc = (blk == 0 && kk == 0) ? 0u : 1u;
          mma(dacc, da, sdesc_sw128(sb + kk * 32, 16, 1024), kIdMain, acc);
          mma(tbase + 256, da, sdesc_sw128(sam + kk * 32, 16, 1024), kIdT, acc);
        }
        commit(&empty[rp.stage]);
        rp.next(S);
        return true;
      };
      uint32_t it = 0;
      if constexpr (C::kDropEpi) {
        // Ring order (the producer's): L(t0), main(t0)[0, h), L(t1),
        // main(t0)[h, n), main(t1)[0, h), L(t2), ...  L(t) goes into t's
        // buffer once the epilogue has drained it; the main blocks of t wait
        // until the epilogue warps have zeroed the dropped entries of L(t).
        const int h = nmain / 2;
        auto lora_into = [&](uint32_t i) -> bool {      // L of the unit's i-th tile
          const uint32_t b = i & 1u, u = i >> 1;
          if (!wait_bar<kPair>(&acc_empty[b], (u & 1u) ^ 1u, ctl)) return false;
          tc_fence_after();
          for (int lb = 0; lb < nlora; ++lb)
            if (!take(nmain + lb, tbase + b * 256)) return false;
          commit(&lora_done[b]);
          return true;
        };
        bool ok = true;
        for (int t = unit; t < p.num_tiles && ok; t += nunits, ++it) {
          const uint32_t buf = it & 1u;
          const uint32_t use = it >> 1;
          const uint32_t dacc = tbase + buf * 256;
          if (t == unit) ok = lora_into(it);
          if (ok) ok = wait_bar<kPair>(&masked[buf], use & 1u, ctl);
          tc_fence_after();
          for (int blk = 0; blk < h && ok; ++blk) ok = take(blk, dacc);
          if (ok && t + nunits < p.num_tiles) ok = lora_into(it + 1);
          for (int blk = h; blk < nmain && ok; ++blk) ok = take(blk, dacc);
          if (ok) commit(&acc_full[buf]);
        }
      } else {
        for (int t = unit; t < p.num_tiles; t += nunits, ++it) {
          const uint32_t buf = it & 1u;
          const uint32_t use = it >> 1;        // how many times this buffer was used before
          if (!wait_bar<kPair>(&acc_empty[buf], (use & 1u) ^ 1u, ctl)) break;
          tc_fence_after();
          const uint32_t dacc = tbase + buf * 256;
          bool ok = true;
          if (C::kTFused && (!p.t_shared || t < p.m_tiles)) {
            for (int blk = 0; blk < nmain && ok; ++blk) ok = take_t(blk, dacc);
            // T is complete once these MMAs retire; the epilogue warps turn it
            // into the LoRA block's operand in shared memory.  (A unit has at
            // most one T tile, its first, so both barriers complete once.)
            if (ok) commit(t_done);
            if (ok) ok = wait_bar<kPair>(t_ready, 0u, ctl);
            tc_fence_after();
          } else {
            for (int blk = 0; blk < nmain && ok; ++blk) ok = take(blk, dacc);
          }
          for (int blk = nmain; blk < nmain + nlora && ok; ++blk) ok = take(blk, dacc);
          if (!ok) break;
          commit(&acc_full[buf]);
        }
      }
      if constexpr (kPair) mma_commit_pair(mma_done, 0x1);
      else mma_commit(mma_done);
      volatile uint32_t zero = 0u;
      AbortCtl quiet{&zero, nullptr};
      wait_bar<kPair>(mma_done, 0, quiet);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..7
    const int q = warp & 3;                  // TMEM lane quadrant
    const int h = ew >> 2;                   // column half
    const int row_in_tile = q * 32 + lane;
    const uint64_t pol_out = l2_policy_evict_first();
    uint32_t acc_empty_addr[2];
#pragma unroll
    for (int b = 0; b < 2; ++b)
      acc_empty_addr[b] = kPair ? mapa_shared(smem_u32(&acc_empty[b]), 0) : smem_u32(&acc_empty[b]);
    // Dropout: in the accumulator buffer of the unit's i-th tile (tile tt),
    // keep the LoRA term m * (s'U A) where this thread's row keeps the
    // element and zero it elsewhere; 16 columns per TMEM load / store.
    auto mask_pass = [&](int tt, uint32_t i) -> bool {
      const uint32_t b = i & 1u, u = i >> 1;
      int mt2, nt2;
      mma_tile_coords(tt, p, mt2, nt2);
      const int row2 = mt2 * C::kTileM + 128 * static_cast<int>(crank) + row_in_tile;
      const bool ok_row = row2 < p.M;
      const int ldm = p.N / 8;
      const bool vec = (reinterpret_cast<uintptr_t>(p.drop.mask) % 16) == 0 && ldm % 16 == 0;
      uint32_t keep[4];
      load_keep_bytes<16>(p.drop.mask + static_cast<size_t>(ok_row ? row2 : 0) * ldm, (nt2 * 256 + h * 128) / 8, ldm,
                          ok_row, vec, keep);
      if (!wait_bar<kPair>(&lora_done[b], u & 1u, ctl)) return false;
      tc_fence_after();
      __syncwarp();
      const uint32_t tl2 = tbase + b * 256 + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
#pragma unroll 1
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t v[16];
        tmem_ld16(tl2 + 16 * c16, v);
        tmem_wait_ld();
        const uint32_t mb = (keep[c16 >> 1] >> (16 * (c16 & 1))) & 0xFFFFu;   // keep bytes 2 c16, 2 c16 + 1
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = ((mb >> j) & 1u) ? v[j] : 0u;
        tmem_st16(tl2 + 16 * c16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&masked[b]), 0));
        else mbar_arrive(&masked[b]);
      }
      return true;
    };
    uint32_t it = 0;
    for (int t = unit; t < p.num_tiles; t += nunits, ++it) {
      int mt, nt;
      mma_tile_coords(t, p, mt, nt);
      const uint32_t buf = it & 1u;
      const uint32_t use = it >> 1;
      const int row = mt * C::kTileM + 128 * static_cast<int>(crank) + row_in_tile;
      const bool row_ok = row < p.M;
      if constexpr (C::kDropEpi) {
        // Zero the dropped entries of the LoRA term before the main blocks
        // accumulate on it: the unit's first tile's term before anything
        // else, the next tile's (in the other buffer) before this tile's
        // epilogue, which the MMA warp needs next.
        bool okm = true;
        if (t == unit) okm = mask_pass(t, it);
        if (okm && t + nunits < p.num_tiles) okm = mask_pass(t + nunits, it + 1);
        if (!okm) break;
      }
      if constexpr (C::kTFused) {
        // Fused T: once a T tile's main K-loop has retired, the column-half-0
        // warps read this row's T from tensor memory, save it in fp32 (the
        // N-tile-0 unit only; without a shared T every unit of the row block
        // computes the same T) and write bf16(s T) as row row_in_tile of the
        // LoRA block's A operand: the A area of the stage the LoRA block
        // occupies (the T tile is the unit's first, so its blocks are the
        // ring's first: the main K-blocks, then the LoRA block),
        // SWIZZLE_128B, 16-byte chunk c at position c ^ (row & 7).  With a
        // shared T they also store bf16(s T) to st_out and then set this
        // warp's flag bit for the row block.
        if (h == 0 && (!p.t_shared || t < p.m_tiles)) {
          if (!wait_bar<kPair>(t_done, 0u, ctl)) break;
          tc_fence_after();
          __syncwarp();
          uint4* lrow = reinterpret_cast<uint4*>(smem + static_cast<uint32_t>(C::kKPairs * nkb % S) * C::kStageBytes +
                                                 row_in_tile * 128);
          const uint32_t tlT = tbase + 256 + (static_cast<uint32_t>(q * 32) << 16);
          const bool wr = p.t_save != nullptr && nt == 0 && row_ok;
          const bool pub = p.t_shared && row_ok;
          for (int c0 = 0; c0 < p.rp; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(tlT + static_cast<uint32_t>(c0), v);
            tmem_wait_ld();
            if (wr) {
              float* dst = p.t_save + static_cast<size_t>(row) * p.r + c0;
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                if (c0 + c < p.r)
                  *reinterpret_cast<float4*>(dst + c) = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                                    __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = p.lora_scale * __uint_as_float(v[8 * hh + e]);
              uint4 pk;
              pk.x = pack_bf16x2(f[0], f[1]);
              pk.y = pack_bf16x2(f[2], f[3]);
              pk.z = pack_bf16x2(f[4], f[5]);
              pk.w = pack_bf16x2(f[6], f[7]);
              lrow[((c0 >> 3) + hh) ^ (row_in_tile & 7)] = pk;
              if (pub && c0 + 8 * hh < p.r)
                *reinterpret_cast<uint4*>(p.st_out + static_cast<size_t>(row) * p.r + c0 + 8 * hh) = pk;
            }
          }
          fence_proxy_async_smem();     // the tensor core reads the operand through the async proxy
          if (p.t_shared) {
            // other CTAs read st_out through TMA (the async proxy)
            fence_proxy_async_global();
            __threadfence();
          }
          tc_fence_before();            // the T columns are rewritten by this unit's next tile
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(t_ready), 0));
            else mbar_arrive(t_ready);
            if (p.t_shared) {
              const int bit = (mt * C::kCtas + static_cast<int>(crank)) * 4 + q;
              red_or_release_gpu(p.t_flags + 1 + bit / 32, 1u << (bit % 32));
            }
          }
        }
      }
      if (!wait_bar<kPair>(&acc_full[buf], use & 1u, ctl)) break;
      tc_fence_after();
      __syncwarp();   // tcgen05.ld is .sync.aligned
      const uint32_t tl = tbase + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
      auto release_acc = [&]() {   // every lane's tcgen05.ld has completed (tmem_wait_ld)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_cluster(acc_empty_addr[buf]);
          else mbar_arrive(&acc_empty[buf]);
        }
      };
      if constexpr (C::kSwigluFwd || kEpi == kMEpiSilu) {
        // Two halves of this thread's columns (SiLU: 64 + 64 of its 128;
        // SwiGLU: 32 + 32 gate columns with their up columns), so that only 64
        // accumulator values are live at a time.  Each flush is one box of the
        // warp's 32 rows x 128 bytes (32 fp32 Z or 64 bf16 Y columns): into
        // its 4 KB slot of shared memory (16-byte chunk j of row r at
        // j ^ (r & 7)), then one TMA store at column x, clipped at the last
        // row and column.
        const int row0 = row - lane;                 // first row of this warp's 32
        uint4* stg = reinterpret_cast<uint4*>(epi_stage + ew * 4096);
        auto flush = [&](const uint4 (&mine)[8], const CUtensorMap* tm, int x) {
          if (lane == 0) bulk_wait_read_all();       // the slot's previous box has been read out
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) stg[lane * 8 + (j ^ (lane & 7))] = mine[j];
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.M && x < p.N) {
            tma_store_2d_hint(tm, stg, x, row0, pol_out);
            bulk_commit_group();
          }
        };
        const int col0 = C::kSwigluFwd ? nt * 128 + h * 64 : nt * 256 + h * 128;
        uint32_t ylo[16];                            // SwiGLU: packed bf16 Y of the first half
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          uint32_t v[64];
          if constexpr (C::kSwigluFwd) {
            tmem_ld32(tl + h * 64 + 32 * hv, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));          // gate
            tmem_ld32(tl + 128 + h * 64 + 32 * hv, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));   // up
          } else {
            tmem_ld32(tl + h * 128 + 64 * hv, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(tl + h * 128 + 64 * hv + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          }
          tmem_wait_ld();
          if (hv == 1) release_acc();
          if (p.z_save != nullptr) {
            // fp32 Z, 32 columns per flush: SwiGLU gate then up; SiLU two column runs
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              const int zc0 = C::kSwigluFwd ? col0 + 32 * hv : col0 + 64 * hv + 32 * part;
              uint4 mine[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int c = part * 32 + 4 * j;
                mine[j] = make_uint4(v[c], v[c + 1], v[c + 2], v[c + 3]);
              }
              flush(mine, &p.tm_z[C::kSwigluFwd ? part : 0], zc0);
            }
          }
          if constexpr (C::kSwigluFwd) {
            // bf16 Y = SiLU(gate) * up: 32 columns per half, one 64-column flush
            uint32_t y[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float yy[2];
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                const float g = __uint_as_float(v[2 * e + k]);
                const float u = __uint_as_float(v[32 + 2 * e + k]);
                yy[k] = g / (1.0f + expf(-g)) * u;
              }
              y[e] = pack_bf16x2(yy[0], yy[1]);
            }
            if (hv == 0) {
#pragma unroll
              for (int e = 0; e < 16; ++e) ylo[e] = y[e];
            } else {
              uint4 mine[8];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                mine[j] = make_uint4(ylo[4 * j], ylo[4 * j + 1], ylo[4 * j + 2], ylo[4 * j + 3]);
                mine[4 + j] = make_uint4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
              }
              flush(mine, &p.tm_out, col0);
            }
          } else {
            // bf16 Y = SiLU(z): 64 columns per half, one flush
            uint4 mine[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float yv[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float z = __uint_as_float(v[8 * j + e]);
                yv[e] = z / (1.0f + expf(-z));
              }
              mine[j].x = pack_bf16x2(yv[0], yv[1]);
              mine[j].y = pack_bf16x2(yv[2], yv[3]);
              mine[j].z = pack_bf16x2(yv[4], yv[5]);
              mine[j].w = pack_bf16x2(yv[6], yv[7]);
            }
            flush(mine, &p.tm_out, col0 + 64 * hv);
          }
        }
      } else if constexpr (kEpi == kMEpiRope || kEpi == kMEpiRopeT) {
        // Identity plus the rotary embedding.  This thread's 128 columns start
        // at a multiple of 128, so they hold whole heads (half = 64: one head,
        // pairs (c, c + 64); half = 32: two heads, pairs (c, c + 32) in each).
        // Two passes, each loading 32 columns at c0 and 32 at c0 + half, so
        // that a pass holds 32 whole pairs: u[e], u[e + 32].
        const int half = p.rope.half;
        const int pr = row_ok ? __ldg(p.rope.pos + row) : 0;
        const bool turn = row_ok && pr >= 0 && pr < p.rope.n_pos;
        if (row_ok && !turn && p.status) atomicOr(p.status, kStatusBadArgument);   // left unturned
        const size_t trow = static_cast<size_t>(turn ? pr : 0) * half;
        const int col0 = nt * 256 + h * 128;
        // Each 32-column group leaves as one box: packed to bf16 in half
        // `part` of the warp's 4 KB slot (row r at 64 r bytes, 16-byte chunk
        // j at position j ^ ((r >> 1) & 3): the 64-byte swizzle of the
        // tensor map), then one TMA store, clipped at the last row and
        // column.  Rows past M carry zeros (their inputs were zero-filled)
        // and are clipped.
        uint4* stg = reinterpret_cast<uint4*>(epi_stage + ew * 4096);
        const int row0 = row - lane;
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          const int c0 = half == 64 ? 32 * hv : 64 * hv;
          uint32_t u[64];
          __syncwarp();   // tcgen05.ld is .sync.aligned
          tmem_ld32(tl + h * 128 + c0, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(tl + h * 128 + c0 + half, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld();
          if (hv == 1) release_acc();
          const int toff = c0 % half;
          if (turn) rope_rotate32(u, p.rope.cos + trow + toff, p.rope.sin + trow + toff);
          if (lane == 0) bulk_wait_read_all();   // both halves of the slot have been read out
          __syncwarp();
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t* w = &u[32 * part + 8 * j];
              uint4 pk;
              pk.x = pack_bf16x2(__uint_as_float(w[0]), __uint_as_float(w[1]));
              pk.y = pack_bf16x2(__uint_as_float(w[2]), __uint_as_float(w[3]));
              pk.z = pack_bf16x2(__uint_as_float(w[4]), __uint_as_float(w[5]));
              pk.w = pack_bf16x2(__uint_as_float(w[6]), __uint_as_float(w[7]));
              stg[part * 128 + lane * 4 + (j ^ ((lane >> 1) & 3))] = pk;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.M) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              const int cc = col0 + c0 + part * half;
              if (cc < p.N) tma_store_2d_hint(&p.tm_out, stg + part * 128, cc, row0, pol_out);
            }
            bulk_commit_group();
          }
        }
      } else if constexpr (kEpi == kMEpiGradF32 || kEpi == kMEpiGradF16F32) {
        // fp32 dX, written or added to (several projections' input gradients
        // summed in a fixed order, one launch after another).  Each 32-column
        // chunk of the warp's 32 rows goes into its 4 KB slot of shared
        // memory (16-byte chunk j of row rr at j ^ (rr & 7), the 128-byte
        // swizzle of the fp32 tensor map) and leaves as one TMA store, or
        // with out_acc one TMA reduce-add (the addition done at L2, one per
        // element and launch), clipped at the last row and column.
        const int row0 = row - lane;                 // first row of this warp's 32
        float4* stg = reinterpret_cast<float4*>(epi_stage + ew * 4096);
        const int col0 = nt * 256 + h * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tl + h * 128 + 32 * c, v);
          tmem_wait_ld();
          if (c == 3) release_acc();
          if (lane == 0) bulk_wait_read_all();       // the slot's previous box has been read out
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            stg[lane * 8 + (j ^ (lane & 7))] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                           __uint_as_float(v[4 * j + 2]),
                                                           __uint_as_float(v[4 * j + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          const int cb = col0 + 32 * c;
          if (lane == 0 && row0 < p.M && cb < p.N) {
            if (p.out_acc) tma_reduce_add_2d_hint(&p.tm_out, stg, cb, row0, pol_out);
            else tma_store_2d_hint(&p.tm_out, stg, cb, row0, pol_out);
            bulk_commit_group();
          }
        }
      } else if constexpr (kEpi == kMEpiCeFwd || kEpi == kMEpiCeFwdZ) {
        // This thread's token row and 128 vocabulary columns [col0, col0 + 128):
        // a running max and sum of exp(z - max) over four 32-column loads
        // (columns past N count as -inf), and z[label] if the label is here.
        // kMEpiCeFwdZ also stores the fp32 logits, row-major [M x N] at
        // out_f32 (the fused forward + backward turns them into the gradient).
        const int col0 = nt * 256 + h * 128;
        const int lab = row_ok ? __ldg(p.ce.labels + row) : -1;
        float mx = -INFINITY, se = 0.0f, zl = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tl + h * 128 + 32 * c, v);
          tmem_wait_ld();
          if (c == 3) release_acc();
          const int cb = col0 + 32 * c;
          if constexpr (kEpi == kMEpiCeFwdZ) {
            // the warp's 32 rows x 32 columns of fp32 logits: into its 4 KB
            // slot (row r at 128 r bytes, 16-byte chunk j at j ^ (r & 7)),
            // then one TMA store, clipped at the last row and column
            uint4* stg = reinterpret_cast<uint4*>(epi_stage + ew * 4096);
            const int row0 = row - lane;
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              stg[lane * 8 + (j ^ (lane & 7))] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && row0 < p.M && cb < p.N) {
              tma_store_2d_hint(&p.tm_out, stg, cb, row0, pol_out);
              bulk_commit_group();
            }
          }
          float cm = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float z = (cb + i < p.N) ? __uint_as_float(v[i]) : -INFINITY;
            v[i] = __float_as_uint(z);
            cm = fmaxf(cm, z);
            if (cb + i == lab) zl = z;
          }
          if (cm == -INFINITY) continue;            // the whole chunk is past N
          const float nm = fmaxf(mx, cm);
          se *= __expf(mx - nm);                    // exp(-inf) = 0 on the first chunk
#pragma unroll
          for (int i = 0; i < 32; ++i) se += __expf(__uint_as_float(v[i]) - nm);
          mx = nm;
        }
        if (row_ok) {
          p.ce.part[static_cast<size_t>(nt * 2 + h) * p.M + row] = make_float2(mx, se);
          if (lab >= col0 && lab < col0 + 128 && lab < p.N) p.ce.zlab[row] = zl;
        }
      } else if constexpr (kEpi == kMEpiCeGrad) {
        // (exp(z - lse) - [column == label]) * scale for this thread's row and
        // 128 columns, bf16, in four 32-column pieces; ignored tokens give 0.
        const int col0 = nt * 256 + h * 128;
        const int lab = row_ok ? __ldg(p.ce.labels + row) : -1;
        const float lse = row_ok ? __ldg(p.ce.lse + row) : 0.0f;
        const float sc = (row_ok && lab >= 0 && lab < p.N) ? __ldg(p.ce.scale) : 0.0f;
        const size_t base = static_cast<size_t>(row) * p.N + col0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tl + h * 128 + 32 * c, v);
          tmem_wait_ld();
          if (c == 3) release_acc();
          if (!row_ok) continue;
          const int cb = col0 + 32 * c;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            float g[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float pz = __expf(__uint_as_float(v[j + e]) - lse);
              g[e] = (pz - (cb + j + e == lab ? 1.0f : 0.0f)) * sc;
            }
            uint4 pk;
            pk.x = pack_bf16x2(g[0], g[1]);
            pk.y = pack_bf16x2(g[2], g[3]);
            pk.z = pack_bf16x2(g[4], g[5]);
            pk.w = pack_bf16x2(g[6], g[7]);
            if (cb + j < p.N) st_global_v4_hint(p.out + base + 32 * c + j, pk, pol_out);
          }
        }
      } else {
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tl + h * 128 + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
        tmem_wait_ld();
        release_acc();
        const int col0 = nt * 256 + h * 128;
        if constexpr (C::kTmaOut) {
          // This warp's 32 rows x 128 columns leave as two 64-column boxes:
          // packed to bf16 in its 4 KB slot of shared memory (row r at 128 r
          // bytes, 16-byte chunk j at position j ^ (r & 7): the 128-byte
          // swizzle the tensor map expects), then one TMA store per box,
          // clipped at the tensor's last row and column.
          uint4* stg = reinterpret_cast<uint4*>(epi_stage + ew * 4096);
          const int row0 = row - lane;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (lane == 0) bulk_wait_read_all();   // the slot's previous box has been read out
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = 64 * k + 8 * j;
              uint4 pk;
              pk.x = pack_bf16x2(__uint_as_float(v[c]), __uint_as_float(v[c + 1]));
              pk.y = pack_bf16x2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
              pk.z = pack_bf16x2(__uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
              pk.w = pack_bf16x2(__uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
              stg[lane * 8 + (j ^ (lane & 7))] = pk;
            }
            fence_proxy_async_smem();              // the TMA engine reads the slot through the async proxy
            __syncwarp();
            if (lane == 0 && row0 < p.M && col0 + 64 * k < p.N) {
              tma_store_2d_hint(&p.tm_out, stg, col0 + 64 * k, row0, pol_out);
              bulk_commit_group();
            }
          }
        } else {
          if (!row_ok) continue;
          const size_t base = static_cast<size_t>(row) * p.N + col0;
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(v[c]), __uint_as_float(v[c + 1]));
            pk.y = pack_bf16x2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
            pk.z = pack_bf16x2(__uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
            pk.w = pack_bf16x2(__uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
            if (col0 + c < p.N) st_global_v4_hint(p.out + base + c, pk, pol_out);
          }
        }
      }
    }
    if constexpr (C::kTmaOut || C::kTmaZ || C::kTmaRope || C::kTmaAct) {
      if (lane == 0) bulk_wait_all();   // this warp's stores are complete before the CTA exits
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();
  if constexpr (C::kTFused) {
    // Shared T: the last CTA to get here (every other CTA is done with the
    // flags) zeroes them for the next launch.
    if (p.t_shared && threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.t_flags, 1u) == gridDim.x - 1) {
        for (int i = 1; i <= kTFlagWords; ++i) atomicExch(p.t_flags + i, 0u);
        atomicExch(p.t_flags, 0u);
      }
    }
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tbase, C::kTmemCols);
    else tmem_dealloc(tbase, C::kTmemCols);
  }
}

}  // namespace lora
