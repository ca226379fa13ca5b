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
//
// A token is valid when 0 <= label < V; label < 0 marks a token to ignore.  A
// label >= V is an argument error: status bit 0x2, and the token is ignored.
#pragma once

#include "sm100.cuh"

namespace lora {

constexpr int kCeMeanThreads = 1024;

__global__ void __launch_bounds__(256) ce_combine_kernel(const float2* __restrict__ part, int nblk, int M, int V,
                                                         const int32_t* __restrict__ labels,
                                                         const float* __restrict__ zlab, float* __restrict__ lse,
                                                         float* __restrict__ loss_tok, uint32_t* status) {
  grid_dep_wait();
  for (int m = blockIdx.x * blockDim.x + threadIdx.x; m < M; m += gridDim.x * blockDim.x) {
    // one pass, rescaling the running sum whenever the maximum grows
    float mx = -INFINITY, se = 0.0f;
    for (int b = 0; b < nblk; ++b) {
      const float2 q = part[static_cast<size_t>(b) * M + m];
      if (q.x == -INFINITY) continue;        // a block wholly past V
      if (q.x > mx) {
        se = se * expf(mx - q.x) + q.y;
        mx = q.x;
      } else {
        se += q.y * expf(q.x - mx);
      }
    }
    const float l = mx + logf(se);
    lse[m] = l;
    const int lab = labels[m];
    if (lab >= V && status) atomicOr(status, kStatusBadArgument);
    loss_tok[m] = (lab >= 0 && lab < V) ? l - zlab[m] : 0.0f;
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

}  // namespace lora
