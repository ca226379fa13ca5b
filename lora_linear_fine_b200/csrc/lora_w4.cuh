// lora_w4.cuh — the 4-bit frozen base weight ("w4g64"): codes q in 0..15 two
// per byte (low nibble = even input feature), one bf16 scale per output row
// and 64 input features stored group-major [d_in/64 x d_out]; the weight value
// is bf16(scale * (q - 8)), rounded to nearest even (the product is exact in
// fp32, so that rounding is the only step).
//
// dequant_w4_kernel writes the bf16 weight for the tiled GEMM path (many
// tokens: the weight is read many times, so it is expanded once).  The
// few-token forward dequantises inside its stream instead (lora_small_m.cuh).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace lora {

constexpr int kW4Group = 64;

// The two weights of one code byte (low nibble = even feature, in the low
// half), as packed bf16: the nibbles become the bf16 numbers 128 + q (the
// exponent of 128 has a 7-bit significand step of 1), 136 is subtracted
// exactly, and one bf16x2 multiply by the scale rounds the exact product to
// nearest even.  The low byte of x holds the codes.
__device__ __forceinline__ uint32_t w4_pair(uint32_t x, __nv_bfloat162 scale2) {
  const uint32_t b = x & 0xFFu;
  const uint32_t y = ((b | (b << 12)) & 0x000F000Fu) | 0x43004300u;   // {128 + q_lo, 128 + q_hi}
  const __nv_bfloat162 off = __floats2bfloat162_rn(136.0f, 136.0f);
  const __nv_bfloat162 v = __hmul2(__hsub2(*reinterpret_cast<const __nv_bfloat162*>(&y), off), scale2);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Eight weights from one 32-bit word of codes (bytes in memory order).
__device__ __forceinline__ uint4 w4_word(uint32_t w, __nv_bfloat162 scale2) {
  return make_uint4(w4_pair(w, scale2), w4_pair(w >> 8, scale2), w4_pair(w >> 16, scale2), w4_pair(w >> 24, scale2));
}

// One thread per 16 codes (8 bytes in, 32 bytes out), grid-stride; consecutive
// threads walk a row, so loads and stores are coalesced.
__global__ void __launch_bounds__(256) dequant_w4_kernel(const uint8_t* __restrict__ Wq,
                                                         const __nv_bfloat16* __restrict__ Ws, long long d_out,
                                                         int d_in, __nv_bfloat16* __restrict__ W) {
  grid_dep_wait();
  const int per_row = d_in / 16;
  const long long n_items = d_out * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_items;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long n = i / per_row;
    const int j = static_cast<int>(i - n * per_row);               // codes 16 j .. 16 j + 15
    const uint2 b = *reinterpret_cast<const uint2*>(Wq + n * (d_in / 2) + 8 * j);
    const __nv_bfloat162 sc2 = __bfloat162bfloat162(Ws[static_cast<long long>((16 * j) / kW4Group) * d_out + n]);
    uint4* dst = reinterpret_cast<uint4*>(W + n * d_in + 16 * j);
    dst[0] = w4_word(b.x, sc2);
    dst[1] = w4_word(b.y, sc2);
  }
}

// Tiled layout of the codes for the few-token kernel: the codes of each
// 128-row x 64-feature tile are 4096 contiguous bytes (row i of the tile at
// 32 i, the nibble order of the row-major format), tiles ordered by 128-row
// slice, then by 64-feature block: tile (g, kb) starts at (g * d_in/64 + kb) *
// 4096.  Rows past d_out (in the last slice) are zero.  One 4 KB bulk copy
// then brings a stage's codes, instead of 128 separate 32-byte row pieces.
constexpr int kW4TileBytes = 128 * 32;

// One thread per 16 bytes of the tiled output, grid-stride.
__global__ void __launch_bounds__(256) tile_w4_kernel(const uint8_t* __restrict__ Wq, long long d_out, int d_in,
                                                      uint8_t* __restrict__ Wt) {
  grid_dep_wait();
  const int nkb = d_in / kW4Group;
  const long long slices = (d_out + 127) / 128;
  const long long n16 = slices * nkb * (kW4TileBytes / 16);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long tile = i / (kW4TileBytes / 16);
    const int within = static_cast<int>(i - tile * (kW4TileBytes / 16));   // 16-byte piece: row within / 2, half within % 2
    const long long g = tile / nkb;
    const int kb = static_cast<int>(tile - g * nkb);
    const long long n = g * 128 + within / 2;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < d_out) v = *reinterpret_cast<const uint4*>(Wq + n * (d_in / 2) + kb * 32 + (within & 1) * 16);
    reinterpret_cast<uint4*>(Wt)[i] = v;
  }
}

}  // namespace lora
