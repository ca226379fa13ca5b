// lora_ce.cuh — the small kernels around the output projection fused with the
// cross-entropy loss ("Swift-All一文详解：如何用Liger-Kernel提升训练效率", 2.2 (3):
// the loss is computed together with the last layer's logits, stably, and its
// gradient comes straight from the previous layer's output without the full
// probability distribution).  The logits themselves are produced and reduced
// inside the tcgen05 GEMM's epilogue (lora_mma.cuh, kMEpiCeFwd / kMEpiCeGrad);
// these kernels finish the per-token and per-batch sums in a fixed order:
//
//   ce_combine_kernel   per token: lse = m + log(sum_b s_b exp(m_b - m)) over
//                       the GEMM's (m_b, s_b) block partials; the token's loss
//                       lse - z[label] (0 for an ignored token)
//   ce_mean_kernel      one CTA: the mean of the valid tokens' losses (fp64
//                       accumulation, fixed tree order)
//   ce_scale_kernel     one CTA: d(loss) / (number of valid tokens), the factor
//                       of every gradient entry
//   ce_dz_kernel        the fused forward + backward: the gradient of the loss
//                       with respect to stored fp32 logits, bf16, with the same
//                       arithmetic as the kMEpiCeGrad epilogue
//
// A token is valid when 0 <= label < V; label < 0 marks a token to ignore.  A
// label >= V is an argument error: status bit 0x2, and the token is ignored.
#pragma once

#include "sm100.cuh"

namespace lora {

constexpr int kCeMeanThreads = 1024;

// Merges (max, sum exp(z - max)) partial q into the running (mx, se):
// rescales the running sum whenever the maximum grows; a partial of a block
// wholly past V (max -inf) changes nothing.
__device__ __forceinline__ void ce_merge(float& mx, float& se, float2 q) {
  if (q.x == -INFINITY) return;
  if (q.x > mx) {
    se = se * expf(mx - q.x) + q.y;
    mx = q.x;
  } else {
    se += q.y * expf(q.x - mx);
  }
}

constexpr int kCeCombineTokens = 8;                          // tokens per CTA
constexpr int kCeCombineGroups = 256 / kCeCombineTokens;     // threads per token

// A CTA of 256 threads per 8 tokens: thread (group g, token t) merges the
// blocks g, g + 32, g + 64, ... of its token in that order; then one thread
// per token merges the 32 group results in group order (a fixed order, so the
// result is deterministic) and finishes lse and the token's loss.
__global__ void __launch_bounds__(256) ce_combine_kernel(const float2* __restrict__ part, int nblk, int M, int V,
                                                         const int32_t* __restrict__ labels,
                                                         const float* __restrict__ zlab, float* __restrict__ lse,
                                                         float* __restrict__ loss_tok, uint32_t* status) {
  grid_dep_wait();
  __shared__ float2 grp[kCeCombineGroups][kCeCombineTokens];
  const int t = threadIdx.x % kCeCombineTokens, g = threadIdx.x / kCeCombineTokens;
  for (int m0 = blockIdx.x * kCeCombineTokens; m0 < M; m0 += gridDim.x * kCeCombineTokens) {
    const int m = m0 + t;
    float mx = -INFINITY, se = 0.0f;
    if (m < M) {
      int b = g;
      for (; b + 3 * kCeCombineGroups < nblk; b += 4 * kCeCombineGroups) {
        float2 q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = part[static_cast<size_t>(b + k * kCeCombineGroups) * M + m];
#pragma unroll
        for (int k = 0; k < 4; ++k) ce_merge(mx, se, q[k]);
      }
      for (; b < nblk; b += kCeCombineGroups) ce_merge(mx, se, part[static_cast<size_t>(b) * M + m]);
    }
    grp[g][t] = make_float2(mx, se);
    __syncthreads();
    if (g == 0 && m < M) {
      float tm = -INFINITY, ts = 0.0f;
#pragma unroll 1
      for (int k = 0; k < kCeCombineGroups; ++k) ce_merge(tm, ts, grp[k][t]);
      const float l = tm + logf(ts);
      lse[m] = l;
      const int lab = labels[m];
      if (lab >= V && status) atomicOr(status, kStatusBadArgument);
      loss_tok[m] = (lab >= 0 && lab < V) ? l - zlab[m] : 0.0f;
    }
    __syncthreads();
  }
}

// Fixed-order sum over a CTA of kCeMeanThreads threads (fp64).
__device__ __forceinline__ double ce_block_sum(double v, double* sh) {
  const int t = threadIdx.x;
  sh[t] = v;
  __syncthreads();
  for (int w = kCeMeanThreads / 2; w > 0; w >>= 1) {
    if (t < w) sh[t] += sh[t + w];
    __syncthreads();
  }
  const double r = sh[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kCeMeanThreads) ce_mean_kernel(const float* __restrict__ loss_tok,
                                                                 const int32_t* __restrict__ labels, int M, int V,
                                                                 float* __restrict__ loss) {
  __shared__ double sh[kCeMeanThreads];
  grid_dep_wait();
  double acc = 0.0, cnt = 0.0;
  for (int m = threadIdx.x; m < M; m += kCeMeanThreads) {
    const int lab = labels[m];
    if (lab >= 0 && lab < V) {
      acc += loss_tok[m];
      cnt += 1.0;
    }
  }
  acc = ce_block_sum(acc, sh);
  cnt = ce_block_sum(cnt, sh);
  if (threadIdx.x == 0) *loss = cnt > 0.0 ? static_cast<float>(acc / cnt) : 0.0f;
}

__global__ void __launch_bounds__(kCeMeanThreads) ce_scale_kernel(const int32_t* __restrict__ labels, int M, int V,
                                                                  const float* __restrict__ dloss,
                                                                  float* __restrict__ scale, uint32_t* status) {
  __shared__ double sh[kCeMeanThreads];
  grid_dep_wait();
  double cnt = 0.0;
  bool bad = false;
  for (int m = threadIdx.x; m < M; m += kCeMeanThreads) {
    const int lab = labels[m];
    cnt += (lab >= 0 && lab < V) ? 1.0 : 0.0;
    bad |= lab >= V;
  }
  if (bad && status) atomicOr(status, kStatusBadArgument);
  cnt = ce_block_sum(cnt, sh);
  if (threadIdx.x == 0) *scale = cnt > 0.0 ? static_cast<float>(static_cast<double>(*dloss) / cnt) : 0.0f;
}

// dz[m][v] = (exp(z[m][v] - lse[m]) - [v == label[m]]) * scale, bf16, from
// the fp32 logits z [M x V] (row-major); 0 for an ignored token.  One thread
// per 8 consecutive columns (two 16-byte loads, one 16-byte store), grid
// stride; the expressions are those of the kMEpiCeGrad epilogue, so the
// result is the one the recomputing backward gives.
__global__ void __launch_bounds__(256) ce_dz_kernel(const float* __restrict__ z, int M, int V,
                                                    const int32_t* __restrict__ labels,
                                                    const float* __restrict__ lse, const float* __restrict__ scale,
                                                    __nv_bfloat16* __restrict__ dz) {
  grid_dep_wait();
  const int per_row = V / 8;
  const long long n = static_cast<long long>(M) * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / per_row);
    const int c0 = static_cast<int>(i - static_cast<long long>(m) * per_row) * 8;
    const int lab = __ldg(labels + m);
    const float l = __ldg(lse + m);
    const float sc = (lab >= 0 && lab < V) ? __ldg(scale) : 0.0f;
    const float4* src = reinterpret_cast<const float4*>(z + static_cast<size_t>(m) * V + c0);
    const float4 a = __ldcs(src), b = __ldcs(src + 1);
    const float zz[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float g[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float pz = __expf(zz[e] - l);
      g[e] = (pz - (c0 + e == lab ? 1.0f : 0.0f)) * sc;
    }
    uint4 pk;
    pk.x = pack_bf16x2(g[0], g[1]);
    pk.y = pack_bf16x2(g[2], g[3]);
    pk.z = pack_bf16x2(g[4], g[5]);
    pk.w = pack_bf16x2(g[6], g[7]);
    *reinterpret_cast<uint4*>(dz + static_cast<size_t>(m) * V + c0) = pk;
  }
}

}  // namespace lora
