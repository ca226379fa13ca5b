// lora_dropout.cuh — dropout on the input of the LoRA branch.
//
// With a {0,1} mask m (one bit per element of X, given by the caller) and
// drop probability p, the adapter sees X_d = X * m / (1 - p) while the frozen
// path sees X.  Writing X_m = X * m (exact in bf16: each element is kept or
// zeroed) and s' = s / (1 - p), the layer is the plain one with the adapter
// input X_m and the scale s':
//   Z  = X W^T + s' (X_m A^T) B^T
//   dA = s' U^T X_m,   dB = s' dZ^T (X_m A^T),   U = dZ B
//   dX = dZ W + m * (s' U A)
// X_m is never stored: the rank passes that read X for the adapter (T and
// dA) zero the dropped elements of their X tiles in shared memory.  Only the
// LoRA term of dX needs the mask outside them.  With one projection the dX
// GEMM forms s' U A in its accumulator first, zeroes its dropped entries in
// tensor memory and accumulates dZ W on top (lora_mma.cuh, kMEpiGradDrop);
// with SwiGLU (two masks on one accumulator) the GEMM runs without its LoRA
// K-blocks and dx_dropout_kernel, below, adds m * (s' U A) afterwards.
//
// Mask layout: [M x d_in/8] bytes, bit j of byte b (least significant first)
// keeps element 8 b + j.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace lora {

struct DxDropoutJob {
  const uint8_t* mask;          // [M x d_in/8]
  const __nv_bfloat16* ut_hi;   // (s' U)^T hi [r x ld]
  const __nv_bfloat16* ut_lo;   // (s' U)^T lo [r x ld]
  const __nv_bfloat16* A;       // [r x d_in]
};

constexpr int kDxRows = 64, kDxCols = 128, kDxRowsPerThread = kDxRows / 16;

// Dynamic shared memory of dx_dropout_kernel for rank r: the rows' s'U
// (fp32, stride r + 1) and the tile's columns of A (bf16).
inline size_t dx_dropout_smem_bytes(int r) {
  return (static_cast<size_t>(kDxRows) * (r + 1) * 4 + 15) / 16 * 16 + static_cast<size_t>(r) * kDxCols * 2;
}

// dX += sum_j m_j * ((s' U_j) A_j) for one or two projections, in place on the
// bf16 dX.  A block takes a 64-row x 128-column tile: it stages the rows'
// s'U (hi + lo, fp32) and the tile's columns of A (bf16) in shared memory
// sized for r.  Each thread owns 8 consecutive columns of 4 rows (16 apart):
// its four 16-byte dX loads and mask bytes are issued before the staging
// barrier, so each thread keeps four independent loads in flight (rows are
// 256 contiguous bytes per 16 threads).
__global__ void __launch_bounds__(256) dx_dropout_kernel(__nv_bfloat16* __restrict__ dX, int M, int d_in, int r,
                                                         int ld, DxDropoutJob j0, DxDropoutJob j1, int np) {
  grid_dep_wait();
  extern __shared__ __align__(16) uint8_t dx_smem[];
  float* sU = reinterpret_cast<float*>(dx_smem);                                   // [kDxRows][r + 1]
  __nv_bfloat16* sA = reinterpret_cast<__nv_bfloat16*>(
      dx_smem + (static_cast<size_t>(kDxRows) * (r + 1) * 4 + 15) / 16 * 16);        // [r][kDxCols]
  const int t = threadIdx.x;
  const int rg = t >> 4, cg = t & 15;         // rows rg + 16 i, columns 8 cg .. 8 cg + 7 of the tile
  const int tiles_m = (M + kDxRows - 1) / kDxRows, tiles_n = d_in / kDxCols + (d_in % kDxCols ? 1 : 0);
  for (long long tile = blockIdx.x; tile < static_cast<long long>(tiles_m) * tiles_n; tile += gridDim.x) {
    const int m0 = static_cast<int>(tile / tiles_n) * kDxRows;
    const int k0 = static_cast<int>(tile % tiles_n) * kDxCols;
    const int k = k0 + 8 * cg;
    float acc[kDxRowsPerThread][8];
    uint4 cur[kDxRowsPerThread];
    uint32_t mb[kDxRowsPerThread][2];
#pragma unroll
    for (int i = 0; i < kDxRowsPerThread; ++i) {
      const int m = m0 + rg + 16 * i;
      cur[i] = make_uint4(0, 0, 0, 0);
      mb[i][0] = mb[i][1] = 0u;
      if (m < M && k < d_in) {
        cur[i] = *reinterpret_cast<const uint4*>(dX + static_cast<size_t>(m) * d_in + k);
        mb[i][0] = j0.mask[static_cast<size_t>(m) * (d_in / 8) + k / 8];
        if (np > 1) mb[i][1] = j1.mask[static_cast<size_t>(m) * (d_in / 8) + k / 8];
      }
    }
#pragma unroll
    for (int i = 0; i < kDxRowsPerThread; ++i) {
      const uint32_t w[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[i][2 * e] = __uint_as_float(w[e] << 16);
        acc[i][2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
    for (int jj = 0; jj < np; ++jj) {
      const DxDropoutJob& J = jj == 0 ? j0 : j1;
      __syncthreads();   // the previous use of sU / sA is over
      for (int i = t; i < kDxRows * r; i += 256) {
        const int c = i / kDxRows, rr = i - c * kDxRows;
        const int mm = m0 + rr;
        float u = 0.0f;
        if (mm < M) {
          const size_t at = static_cast<size_t>(c) * ld + mm;
          u = __bfloat162float(J.ut_hi[at]) + __bfloat162float(J.ut_lo[at]);
        }
        sU[rr * (r + 1) + c] = u;
      }
      for (int i = t; i < r * (kDxCols / 8); i += 256) {
        const int c = i / (kDxCols / 8), q = i - c * (kDxCols / 8);
        const int kk = k0 + 8 * q;
        uint4 a = make_uint4(0, 0, 0, 0);
        if (kk < d_in) a = *reinterpret_cast<const uint4*>(J.A + static_cast<size_t>(c) * d_in + kk);
        *reinterpret_cast<uint4*>(&sA[c * kDxCols + 8 * q]) = a;
      }
      __syncthreads();
      float add[kDxRowsPerThread][8];
#pragma unroll
      for (int i = 0; i < kDxRowsPerThread; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) add[i][e] = 0.0f;
      for (int c = 0; c < r; ++c) {
        const uint4 a = *reinterpret_cast<const uint4*>(&sA[c * kDxCols + 8 * cg]);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        float av[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          av[2 * e] = __uint_as_float(w[e] << 16);
          av[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
#pragma unroll
        for (int i = 0; i < kDxRowsPerThread; ++i) {
          const float u = sU[(rg + 16 * i) * (r + 1) + c];
#pragma unroll
          for (int e = 0; e < 8; ++e) add[i][e] = fmaf(u, av[e], add[i][e]);
        }
      }
#pragma unroll
      for (int i = 0; i < kDxRowsPerThread; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (((jj == 0 ? mb[i][0] : mb[i][1]) >> e) & 1u) acc[i][e] += add[i][e];
    }
#pragma unroll
    for (int i = 0; i < kDxRowsPerThread; ++i) {
      const int m = m0 + rg + 16 * i;
      if (m < M && k < d_in) {
        uint4 o;
        o.x = pack_bf16x2(acc[i][0], acc[i][1]);
        o.y = pack_bf16x2(acc[i][2], acc[i][3]);
        o.z = pack_bf16x2(acc[i][4], acc[i][5]);
        o.w = pack_bf16x2(acc[i][6], acc[i][7]);
        *reinterpret_cast<uint4*>(dX + static_cast<size_t>(m) * d_in + k) = o;
      }
    }
  }
}

}  // namespace lora
