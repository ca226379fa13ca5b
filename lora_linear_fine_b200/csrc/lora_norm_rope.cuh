// lora_norm_rope.cuh — RMSNorm prologue and rotary-embedding epilogue of the
// attention-input (q, k, v) LoRA linears.
//
// The sequence they wrap ("Swift-All一文详解：如何用Liger-Kernel提升训练效率",
// 2.2 (1) "RMSNorm + Rotary Embedding + Attention QKV 融合"):
//   x_n = bf16(x * rstd * g),  rstd = 1 / sqrt(mean(x^2) + eps)   (per token)
//   Z_j = x_n W_j^T + s (x_n A_j^T) B_j^T                         (q, k, v)
//   q = rot(Z_q), k = rot(Z_k), v = Z_v
// rot turns feature i of every head with feature i + h (h = head_dim / 2) by
// the angle whose cosine and sine the caller's tables hold for the token's
// position: (a, b) -> (a c - b s, b c + a s).
//
// * rmsnorm_fwd_kernel writes x_n once; the three projections' forward GEMMs
//   (which also form T) and the backward's dA passes read it.  The sum of
//   squares and rstd are taken in fp64, and x * rstd * g is rounded to bf16
//   from fp32 where that provably gives the same bf16 as the fp64 value (from
//   fp64 elsewhere), so x_n is the correctly rounded norm.
// * The rotation of q and k runs in the forward GEMM's epilogue on the fp32
//   accumulator (rope_rotate32, kMEpiRope in lora_mma.cuh): the pre-rotation
//   values never leave the chip.
// * rope_bwd_kernel turns dY back (dZ = R^T dY) and emits dZ as fp16 hi + lo,
//   the operand form of the backward with an activation.
// * The projections' dX GEMMs write and then add their input gradients into
//   one fp32 dx_n; rmsnorm_bwd_kernel applies the norm's backward:
//   dx = rstd (g dx_n - x_hat mean(g dx_n x_hat)), x_hat = x rstd.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace lora {

constexpr int kNormWarps = 8;      // token rows per CTA: one warp per row
constexpr float kRopeF16Max = 65504.0f;   // largest finite fp16

// Nearest bf16 (ties to even) of a double, without double rounding:
// truncate to fp32 and, when that dropped anything, set the last fp32 bit
// (rounding to odd), then round to nearest even.  fp32 keeps 16 bits more than
// bf16, so the odd bit can decide a tie only in the direction of the dropped
// part (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums:
// proved algorithms using rounding to odd", IEEE Trans. Computers 57(4), 2008).
// Normal range.
__device__ __forceinline__ __nv_bfloat16 bf16_from_f64(double x) {
  float f = __double2float_rz(x);
  if (static_cast<double>(f) != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __float2bfloat16_rn(f);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

// x_n [M x d] bf16 and rstd [M] fp32 from X [M x d] bf16 and g [d] bf16.
// One warp per row, 16-byte loads (8 features per lane and step).  The squares
// of bf16 values are exact in fp64; their sum is exact too unless the row's
// magnitudes span a very wide range, and otherwise off by a relative 2^-53 or
// so, far below the bf16 rounding that follows.  The warp sums its lanes'
// partials by a butterfly, which leaves every lane the same value.  The second
// pass reads the row again (from L1 / L2) to write x_n.
__global__ void __launch_bounds__(32 * kNormWarps)
    rmsnorm_fwd_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ g, long long M, int d,
                       double eps, __nv_bfloat16* __restrict__ Xn, float* __restrict__ rstd) {
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nv = d / 8;
  const uint4* gv = reinterpret_cast<const uint4*>(g);
  for (long long row = blockIdx.x * static_cast<long long>(kNormWarps) + (threadIdx.x >> 5); row < M;
       row += static_cast<long long>(gridDim.x) * kNormWarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + row * d);
    double ss = 0.0;
    for (int c = lane; c < nv; c += 32) {
      float f[8];
      unpack_bf16x8(xr[c], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fma(static_cast<double>(f[e]), static_cast<double>(f[e]), ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double inv = 1.0 / sqrt(ss / static_cast<double>(d) + eps);
    const float inv32 = static_cast<float>(inv);
    if (lane == 0) rstd[row] = inv32;
    uint4* yr = reinterpret_cast<uint4*>(Xn + row * d);
    for (int c = lane; c < nv; c += 32) {
      float f[8], w[8];
      unpack_bf16x8(xr[c], f);
      unpack_bf16x8(__ldg(gv + c), w);
      __align__(16) __nv_bfloat16 o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        // The value to round is y = (x * inv) * g in fp64.  In fp32 (inv
        // rounded to fp32, two products) it is off by at most 3 units in the
        // last place of fp32 (each of the three roundings adds at most half
        // an ulp, relative 2^-24, and an ulp is at least 2^-24 of |y|).  So
        // unless its 16 bits below bf16 precision lie within 16 ulps of
        // 0x8000 (a bf16 rounding midpoint), the fp32 value rounds to the
        // same bf16 as y.  Zero, subnormal and non-finite fp32 values and
        // the near-midpoint ones take the fp64 path.
        const float y = (f[e] * inv32) * w[e];
        const uint32_t b = __float_as_uint(y);
        const uint32_t ex = (b >> 23) & 0xFFu;
        const int low = static_cast<int>(b & 0xFFFFu) - 0x8000;
        if (ex != 0u && ex != 0xFFu && (low > 16 || low < -16)) o[e] = __float2bfloat16_rn(y);
        else o[e] = bf16_from_f64((static_cast<double>(f[e]) * inv) * static_cast<double>(w[e]));
      }
      yr[c] = *reinterpret_cast<const uint4*>(o);
    }
  }
}

// dX [M x d] bf16 = rstd (g dx_n - x_hat mean(g dx_n x_hat)), x_hat = x rstd,
// dx_n [M x d] fp32: the projections' input gradients summed in fp32 by their
// dX GEMMs (three bf16 roundings before the sum would cost the bound on the
// near-zero entries of dx).  One warp per row, fp32, two passes.
__global__ void __launch_bounds__(32 * kNormWarps)
    rmsnorm_bwd_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ g,
                       const float* __restrict__ rstd, const float* __restrict__ dxn, long long M, int d,
                       __nv_bfloat16* __restrict__ dX) {
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nv = d / 8;
  const uint4* gv = reinterpret_cast<const uint4*>(g);
  auto grad8 = [&](long long row, int c, float (&dy)[8]) {
    const float4* q = reinterpret_cast<const float4*>(dxn + row * d) + 2 * c;
    const float4 a = q[0], b = q[1];
    dy[0] = a.x; dy[1] = a.y; dy[2] = a.z; dy[3] = a.w;
    dy[4] = b.x; dy[5] = b.y; dy[6] = b.z; dy[7] = b.w;
  };
  for (long long row = blockIdx.x * static_cast<long long>(kNormWarps) + (threadIdx.x >> 5); row < M;
       row += static_cast<long long>(gridDim.x) * kNormWarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + row * d);
    const float r = rstd[row];
    float dot = 0.0f;
    for (int c = lane; c < nv; c += 32) {
      float x[8], w[8], dy[8];
      unpack_bf16x8(xr[c], x);
      unpack_bf16x8(__ldg(gv + c), w);
      grad8(row, c, dy);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(w[e] * dy[e], x[e] * r, dot);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float mean = dot / static_cast<float>(d);
    uint4* out = reinterpret_cast<uint4*>(dX + row * d);
    for (int c = lane; c < nv; c += 32) {
      float x[8], w[8], dy[8];
      unpack_bf16x8(xr[c], x);
      unpack_bf16x8(__ldg(gv + c), w);
      grad8(row, c, dy);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = r * (w[2 * e] * dy[2 * e] - x[2 * e] * r * mean);
        const float b = r * (w[2 * e + 1] * dy[2 * e + 1] - x[2 * e + 1] * r * mean);
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        ow[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      out[c] = o;
    }
  }
}

// The rotation of 32 pairs held by one epilogue thread: u[e] and u[e + 32] are
// features i and i + half of one head, i = toff + e; cs / sn point at the
// token's table rows plus toff (16-byte aligned).  Unrolled, so that u stays in
// registers.
__device__ __forceinline__ void rope_rotate32(uint32_t (&u)[64], const float* __restrict__ cs,
                                              const float* __restrict__ sn) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 c4 = __ldg(reinterpret_cast<const float4*>(cs + e));
    const float4 s4 = __ldg(reinterpret_cast<const float4*>(sn + e));
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
    const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(u[e + k]);
      const float b = __uint_as_float(u[e + k + 32]);
      u[e + k] = __float_as_uint(a * cc[k] - b * ss[k]);
      u[e + k + 32] = __float_as_uint(b * cc[k] + a * ss[k]);
    }
  }
}

struct RopeTables {
  const int32_t* pos;   // [M] position of each token
  const float* cos;     // [n_pos x half]
  const float* sin;     // [n_pos x half]
  long long n_pos;
  int half;             // head_dim / 2
};

// dZ = R^T dY for a rotated projection, as fp16 hi + lo (lo = fp16(dZ - hi)).
// One thread per (token, head, 8 pairs): two 16-byte loads of dY (features i
// and i + half), the table rows' 8 cosines and sines, four 16-byte stores.  A
// position outside [0, n_pos) sets kStatusBadArgument and passes that token's
// gradient through unturned (as the forward left its output); a value outside
// fp16's range sets kStatusF16Range.
__global__ void __launch_bounds__(256)
    rope_bwd_kernel(const __nv_bfloat16* __restrict__ dY, RopeTables t, long long M, int N,
                    __half* __restrict__ g_hi, __half* __restrict__ g_lo, uint32_t* status) {
  grid_dep_wait();
  const int chunks = t.half / 8;
  const int heads = N / (2 * t.half);
  const long long per_row = static_cast<long long>(heads) * chunks;
  const long long items = M * per_row;
  bool bad_pos = false, bad_range = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < items;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = i / per_row;
    const int rem = static_cast<int>(i - m * per_row);
    const int head = rem / chunks;
    const int ch = rem - head * chunks;
    const long long a0 = m * N + static_cast<long long>(head) * 2 * t.half + ch * 8;
    const long long b0 = a0 + t.half;
    float a[8], b[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(dY + a0), a);
    unpack_bf16x8(*reinterpret_cast<const uint4*>(dY + b0), b);
    float c[8], s[8];
    const int p = t.pos[m];
    if (p >= 0 && p < t.n_pos) {
      const float4* cp = reinterpret_cast<const float4*>(t.cos + static_cast<long long>(p) * t.half + ch * 8);
      const float4* sp = reinterpret_cast<const float4*>(t.sin + static_cast<long long>(p) * t.half + ch * 8);
      const float4 c0 = __ldg(cp), c1 = __ldg(cp + 1), s0 = __ldg(sp), s1 = __ldg(sp + 1);
      c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w; c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
      s[0] = s0.x; s[1] = s0.y; s[2] = s0.z; s[3] = s0.w; s[4] = s1.x; s[5] = s1.y; s[6] = s1.z; s[7] = s1.w;
    } else {
      bad_pos = true;
#pragma unroll
      for (int e = 0; e < 8; ++e) { c[e] = 1.0f; s[e] = 0.0f; }
    }
    __align__(16) __half ah[8], al[8], bh[8], bl[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float ga = a[e] * c[e] + b[e] * s[e];
      const float gb = b[e] * c[e] - a[e] * s[e];
      ah[e] = __float2half_rn(ga);
      al[e] = __float2half_rn(ga - __half2float(ah[e]));
      bh[e] = __float2half_rn(gb);
      bl[e] = __float2half_rn(gb - __half2float(bh[e]));
      if (!(fabsf(ga) <= kRopeF16Max) || !(fabsf(gb) <= kRopeF16Max)) bad_range = true;
    }
    *reinterpret_cast<uint4*>(g_hi + a0) = *reinterpret_cast<const uint4*>(ah);
    *reinterpret_cast<uint4*>(g_lo + a0) = *reinterpret_cast<const uint4*>(al);
    *reinterpret_cast<uint4*>(g_hi + b0) = *reinterpret_cast<const uint4*>(bh);
    *reinterpret_cast<uint4*>(g_lo + b0) = *reinterpret_cast<const uint4*>(bl);
  }
  if (status) {
    if (bad_pos) atomicOr(status, kStatusBadArgument);
    if (bad_range) atomicOr(status, kStatusF16Range);
  }
}

}  // namespace lora
