// lora_linear.cu — the C ABI (include/lora_linear.h): argument checks, the
// workspace layout, tensor-map encoding and the launch sequence of the forward
// and backward of the fused LoRA-adapted linear layer on sm_100a.
#include "lora_linear.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "lora_gemm.cuh"
#include "lora_rank.cuh"
#include "lora_small_m.cuh"

namespace {

using namespace lora;

constexpr int kAbiVersion = 1;
constexpr int kTargetCtas = 148;   // SM count of a B200; sets split-K widths
constexpr size_t kStatusBytes = 256;

// ---------------------------------------------------------------------------
// debug logging (LORA_LINEAR_DEBUG=1)
// ---------------------------------------------------------------------------
bool debug_on() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_DEBUG");
    v = (e && e[0] && e[0] != '0') ? 1 : 0;
  }
  return v == 1;
}
#define LORA_LOG(...)                                  \
  do {                                                 \
    if (debug_on()) {                                  \
      std::fprintf(stderr, "[lora_linear] " __VA_ARGS__); \
      std::fprintf(stderr, "\n");                      \
    }                                                  \
  } while (0)

// ---------------------------------------------------------------------------
// device queries (cached per device)
// ---------------------------------------------------------------------------
struct DevInfo {
  int sms = 0;
  int major = 0;
  int minor = 0;
};

std::mutex g_mu;
DevInfo g_dev[64];
bool g_dev_valid[64] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

lora_status_t device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev_valid[dev]) {
    DevInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return LORA_ERR_CUDA;
    g_dev[dev] = d;
    g_dev_valid[dev] = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return LORA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_dev[dev];
  return LORA_OK;
}

// 2D bf16 tensor map with 128-byte swizzle: `inner` contiguous elements per
// row, `outer` rows `row_elems` elements apart; box = box_inner x box_outer.
bool make_tm(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_elems,
             uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) LORA_LOG("cuTensorMapEncodeTiled failed (%d): inner=%llu outer=%llu box=%ux%u", (int)r,
                                  (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// argument checks and sizes
// ---------------------------------------------------------------------------
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int rank_pad(int64_t r) { return r == 0 ? 0 : (r <= 16 ? 16 : (r <= 32 ? 32 : 64)); }

lora_status_t check_desc(const lora_linear_desc* d) {
  if (d == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->M < 0 || d->d_in <= 0 || d->d_out <= 0 || d->r < 0) return LORA_ERR_INVALID_ARG;
  if (d->act < LORA_ACT_IDENTITY || d->act > LORA_ACT_SWIGLU) return LORA_ERR_INVALID_ARG;
  if (d->M > (int64_t(1) << 31) - 1 || d->d_in > (int64_t(1) << 30) || d->d_out > (int64_t(1) << 30))
    return LORA_ERR_UNSUPPORTED;
  if (d->d_in % 8 != 0 || d->d_out % 8 != 0) return LORA_ERR_ALIGNMENT;
  if (d->r % 8 != 0 || d->r > 64) return LORA_ERR_UNSUPPORTED;
  return LORA_OK;
}

// Split-K width for a rank-r product with `tiles` row tiles and `nkb` 64-wide K blocks.
int rank_splits(int64_t tiles, int64_t nkb) {
  int64_t s = kTargetCtas / (tiles > 0 ? tiles : 1);
  if (s < 1) s = 1;
  if (s > nkb) s = nkb > 0 ? nkb : 1;
  if (s > 64) s = 64;
  return static_cast<int>(s);
}

// Workspace layout of the backward (offsets in bytes, each 256-aligned).
struct BwdLayout {
  size_t bt[2], tw[2], tt_hi[2], tt_lo[2], uw, ut_hi[2], ut_lo[2], dz_hi[2], dz_lo[2];
  size_t part_a, part_b, part_u;
  int splits_a, splits_b, splits_u, splits_t;
  size_t total;
};

size_t fwd_workspace(const lora_linear_desc* d) {
  const int np = d->act == LORA_ACT_SWIGLU ? 2 : 1;
  size_t off = kStatusBytes;
  if (d->r > 0) off += np * align_up(static_cast<size_t>(d->r) * d->d_out * 2, 256);
  return off;
}

BwdLayout bwd_layout(const lora_linear_desc* d) {
  BwdLayout L{};
  const int np = d->act == LORA_ACT_SWIGLU ? 2 : 1;
  const int RP = rank_pad(d->r);
  const int64_t M8 = align_up(static_cast<size_t>(d->M > 0 ? d->M : 1), 8);
  size_t off = kStatusBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  // U of all pairs is one [npair][M x r] block: the dX kernel writes it that way.
  if (d->r > 0) L.uw = take(static_cast<size_t>(np) * d->M * d->r * 4);
  for (int j = 0; j < np; ++j) {
    if (d->r > 0) {
      L.bt[j] = take(static_cast<size_t>(d->r) * d->d_out * 2);
      L.tw[j] = take(static_cast<size_t>(d->M) * d->r * 4);
      L.tt_hi[j] = take(static_cast<size_t>(d->r) * M8 * 2);
      L.tt_lo[j] = take(static_cast<size_t>(d->r) * M8 * 2);
      L.ut_hi[j] = take(static_cast<size_t>(d->r) * M8 * 2);
      L.ut_lo[j] = take(static_cast<size_t>(d->r) * M8 * 2);
    }
    if (d->act != LORA_ACT_IDENTITY) {
      L.dz_hi[j] = take(static_cast<size_t>(d->M) * d->d_out * 2);
      L.dz_lo[j] = take(static_cast<size_t>(d->M) * d->d_out * 2);
    }
  }
  if (d->r > 0) {
    const int64_t tiles_a = ceil_div(d->d_in, 128), tiles_b = ceil_div(d->d_out, 128), tiles_u = ceil_div(d->M, 128);
    const int64_t nkb_tok = ceil_div(d->M, 64);
    L.splits_a = rank_splits(tiles_a, nkb_tok);
    L.splits_b = rank_splits(tiles_b, nkb_tok);
    L.splits_u = rank_splits(tiles_u, ceil_div(d->d_out, 64));
    L.splits_t = rank_splits(tiles_u, ceil_div(d->d_in, 64));
    const int su = L.splits_u > L.splits_t ? L.splits_u : L.splits_t;
    L.part_a = take(static_cast<size_t>(L.splits_a) * tiles_a * 128 * RP * 4);
    L.part_b = take(static_cast<size_t>(L.splits_b) * tiles_b * 128 * RP * 4);
    L.part_u = take(static_cast<size_t>(su) * (tiles_u > 0 ? tiles_u : 1) * 128 * RP * 4);
  }
  L.total = off;
  return L;
}

std::atomic<uint64_t> g_launches{0};

lora_status_t cuda_error(const char* what) {
  const cudaError_t e = cudaGetLastError();
  LORA_LOG("%s: %s", what, cudaGetErrorString(e));
  return LORA_ERR_CUDA;
}

// Called right after every kernel launch.
lora_status_t check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    LORA_LOG("%s: %s", what, cudaGetErrorString(e));
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

// ---------------------------------------------------------------------------
// kernel launchers
// ---------------------------------------------------------------------------
template <bool kBwd, int kRP, int kNPair, int kEpi>
lora_status_t launch_gemm(const GemmParams& p, int sms, cudaStream_t st) {
  using C = GemmCfg<kBwd, kRP, kNPair, kEpi>;
  auto k = lora_gemm_kernel<kBwd, kRP, kNPair, kEpi>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return cuda_error("cudaFuncSetAttribute(gemm)");
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  LORA_LOG("gemm bwd=%d RP=%d npair=%d epi=%d tiles=%d grid=%d smem=%d stages=%d", (int)kBwd, kRP, kNPair, kEpi,
           p.num_tiles, grid, C::kSmemBytes, C::kStages);
  k<<<grid, kGemmThreads, C::kSmemBytes, st>>>(p);
  return check_launch("lora_gemm_kernel");
}

template <bool kBwd, int kNPair, int kEpi>
lora_status_t launch_gemm_rp(int RP, const GemmParams& p, int sms, cudaStream_t st) {
  switch (RP) {
    case 0: return launch_gemm<kBwd, 0, kNPair, kEpi>(p, sms, st);
    case 16: return launch_gemm<kBwd, 16, kNPair, kEpi>(p, sms, st);
    case 32: return launch_gemm<kBwd, 32, kNPair, kEpi>(p, sms, st);
    case 64: return launch_gemm<kBwd, 64, kNPair, kEpi>(p, sms, st);
    default: return LORA_ERR_UNSUPPORTED;
  }
}

template <bool kAMN, int kRP, int kPairs>
lora_status_t launch_rank(const RankGemmParams& p, int splits, cudaStream_t st) {
  using C = RankCfg<kAMN, kRP, kPairs>;
  auto k = rank_gemm_kernel<kAMN, kRP, kPairs>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return cuda_error("cudaFuncSetAttribute(rank)");
  LORA_LOG("rank mn=%d RP=%d pairs=%d rows=%d K=%d tiles=%d splits=%d", (int)kAMN, kRP, kPairs, p.rows, p.K,
           p.m_tiles, splits);
  k<<<p.m_tiles * splits, kRankThreads, C::kSmemBytes, st>>>(p);
  return check_launch("rank_gemm_kernel");
}

template <bool kAMN, int kPairs>
lora_status_t launch_rank_rp(int RP, const RankGemmParams& p, int splits, cudaStream_t st) {
  switch (RP) {
    case 16: return launch_rank<kAMN, 16, kPairs>(p, splits, st);
    case 32: return launch_rank<kAMN, 32, kPairs>(p, splits, st);
    case 64: return launch_rank<kAMN, 64, kPairs>(p, splits, st);
    default: return LORA_ERR_UNSUPPORTED;
  }
}

int grid_for(long long n, int per_block, int sms) {
  long long g = (n + per_block - 1) / per_block;
  if (g > static_cast<long long>(sms) * 8) g = static_cast<long long>(sms) * 8;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

lora_status_t transpose_b(const void* B, int64_t d_out, int64_t r, void* Bt, int sms, cudaStream_t st) {
  const long long n = d_out * r;
  transpose_b_kernel<<<grid_for(n, 256, sms), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(B), (int)d_out,
                                                           (int)r, static_cast<__nv_bfloat16*>(Bt));
  return check_launch("transpose_b_kernel");
}

lora_status_t reduce_partials(const float* part, int splits, int rows, int RP, int r, const float* add, float* dst,
                              int transpose, int sms, cudaStream_t st) {
  const long long n = static_cast<long long>(rows) * r;
  const int rows_pad = static_cast<int>(ceil_div(rows, 128) * 128);
  reduce_partials_kernel<<<grid_for(n, 256, sms), 256, 0, st>>>(part, splits, rows_pad, RP, rows, r, add, dst,
                                                               transpose);
  return check_launch("reduce_partials_kernel");
}

lora_status_t rank_split_t(const float* src, int M, int r, float scale, void* hi, void* lo, int ld, int sms,
                           cudaStream_t st) {
  const long long n = static_cast<long long>(M) * r;
  rank_split_t_kernel<<<grid_for(n, 256, sms), 256, 0, st>>>(src, M, r, scale, static_cast<__nv_bfloat16*>(hi),
                                                             static_cast<__nv_bfloat16*>(lo), ld);
  return check_launch("rank_split_t_kernel");
}

#define LORA_TRY(...)                    \
  do {                                   \
    const lora_status_t _s = (__VA_ARGS__); \
    if (_s != LORA_OK) return _s;        \
  } while (0)

lora_status_t common_checks(const lora_linear_desc* d, void* ws, size_t ws_bytes, size_t need, DevInfo* dev) {
  LORA_TRY(check_desc(d));
  LORA_TRY(device_info(dev));
  if (dev->major != 10 || dev->minor != 0) return LORA_ERR_ARCH;
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return LORA_ERR_WORKSPACE;
  return LORA_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

int lora_linear_abi_version(void) { return kAbiVersion; }

uint64_t lora_linear_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* lora_status_string(lora_status_t s) {
  switch (s) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARG: return "invalid argument";
    case LORA_ERR_ALIGNMENT: return "misaligned pointer or dimension (16-byte pointers, d_in/d_out multiples of 8)";
    case LORA_ERR_UNSUPPORTED: return "unsupported shape (r must be 0 or a multiple of 8 up to 64)";
    case LORA_ERR_ARCH: return "current device is not sm_100 (B200)";
    case LORA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_DEVICE_STATUS: return "device status word is non-zero";
  }
  return "unknown status";
}

size_t lora_linear_workspace_size(const lora_linear_desc* desc, int for_backward) {
  if (check_desc(desc) != LORA_OK) return 0;
  return for_backward ? bwd_layout(desc).total : fwd_workspace(desc);
}

lora_status_t lora_linear_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || workspace_bytes < kStatusBytes) return LORA_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return cuda_error("cudaMemsetAsync");
  return LORA_OK;
}

lora_status_t lora_linear_device_status(const void* workspace, void* stream, uint32_t* out_status) {
  if (workspace == nullptr || out_status == nullptr) return LORA_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return cuda_error("cudaMemcpyAsync(status)");
  if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_error("cudaStreamSynchronize");
  *out_status = v;
  return v == 0 ? LORA_OK : LORA_ERR_DEVICE_STATUS;
}

lora_status_t lora_linear_fwd(const lora_linear_desc* d, const void* X, const void* W, const void* A, const void* B,
                              const void* W_up, const void* A_up, const void* B_up, void* Y, float* T_save,
                              float* Z_save, void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_desc(d));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  const int np = swiglu ? 2 : 1;
  if (X == nullptr || W == nullptr || Y == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->r > 0 && (A == nullptr || B == nullptr)) return LORA_ERR_INVALID_ARG;
  if (swiglu && (W_up == nullptr || (d->r > 0 && (A_up == nullptr || B_up == nullptr)))) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, fwd_workspace(d), &dev));
  if (d->M == 0) return LORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const int RP = rank_pad(d->r);

  if (d->M <= kSmallMMax && d->r > 0 && !swiglu) {
    // Memory-bound small-token path: W streamed once, no B^T copy needed.
    return small_m_forward(d, X, W, A, B, Y, T_save, Z_save, status, dev.sms, st);
  }

  const void* Wp[2] = {W, W_up};
  const void* Ap[2] = {A, A_up};
  const void* Bp[2] = {B, B_up};
  void* Bt[2] = {nullptr, nullptr};
  if (d->r > 0) {
    size_t off = kStatusBytes;
    for (int j = 0; j < np; ++j) {
      Bt[j] = ws + off;
      off += align_up(static_cast<size_t>(d->r) * d->d_out * 2, 256);
      LORA_TRY(transpose_b(Bp[j], d->d_out, d->r, Bt[j], dev.sms, st));
    }
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int outc = swiglu ? 128 : 256;
  bool ok = make_tm(&p.tm_a[0], X, d->d_in, d->M, d->d_in, 64, 128);
  for (int j = 0; j < np; ++j) {
    ok = ok && make_tm(&p.tm_w[j], Wp[j], d->d_in, d->d_out, d->d_in, 64, swiglu ? 128 : 256);
    if (d->r > 0) {
      ok = ok && make_tm(&p.tm_r[j], Ap[j], d->d_in, d->r, d->d_in, 64, RP);
      ok = ok && make_tm(&p.tm_up[j], Bt[j], d->d_out, d->r, d->d_out, 64, RP);
    }
  }
  if (!ok) return LORA_ERR_CUDA;
  p.M = static_cast<int>(d->M);
  p.N = static_cast<int>(d->d_out);
  p.K = static_cast<int>(d->d_in);
  p.r = static_cast<int>(d->r);
  p.s = d->s;
  p.out = static_cast<__nv_bfloat16*>(Y);
  p.rank_save = d->r > 0 ? T_save : nullptr;
  p.z_save = d->act != LORA_ACT_IDENTITY ? Z_save : nullptr;
  p.status = status;
  p.m_tiles = static_cast<int>(ceil_div(d->M, kBM));
  p.n_tiles = static_cast<int>(ceil_div(d->d_out, outc));
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.group_m = 8;
  switch (d->act) {
    case LORA_ACT_IDENTITY: return launch_gemm_rp<false, 1, kEpiIdentity>(RP, p, dev.sms, st);
    case LORA_ACT_SILU: return launch_gemm_rp<false, 1, kEpiSilu>(RP, p, dev.sms, st);
    default: return launch_gemm_rp<false, 2, kEpiSwiglu>(RP, p, dev.sms, st);
  }
}

lora_status_t lora_linear_bwd(const lora_linear_desc* d, const void* dY, const void* X, const void* W, const void* A,
                              const void* B, const void* W_up, const void* A_up, const void* B_up,
                              const float* T_save, const float* Z_save, void* dX, float* dA, float* dB,
                              float* dA_up, float* dB_up, void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_desc(d));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  const int np = swiglu ? 2 : 1;
  if (dY == nullptr || X == nullptr || W == nullptr || dX == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->r > 0 && (A == nullptr || B == nullptr || dA == nullptr || dB == nullptr)) return LORA_ERR_INVALID_ARG;
  if (swiglu && (W_up == nullptr || (d->r > 0 && (A_up == nullptr || B_up == nullptr || dA_up == nullptr ||
                                                  dB_up == nullptr))))
    return LORA_ERR_INVALID_ARG;
  if (d->act != LORA_ACT_IDENTITY && Z_save == nullptr) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  const BwdLayout L = bwd_layout(d);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, L.total, &dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* dAp[2] = {dA, dA_up};
  float* dBp[2] = {dB, dB_up};
  if (d->M == 0) {
    for (int j = 0; j < np && d->r > 0; ++j) {
      if (cudaMemsetAsync(dAp[j], 0, static_cast<size_t>(d->r) * d->d_in * 4, st) != cudaSuccess ||
          cudaMemsetAsync(dBp[j], 0, static_cast<size_t>(d->r) * d->d_out * 4, st) != cudaSuccess)
        return cuda_error("cudaMemsetAsync");
    }
    return LORA_OK;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const int RP = rank_pad(d->r);
  const int M = static_cast<int>(d->M);
  const int r = static_cast<int>(d->r);
  const int M8 = static_cast<int>(align_up(static_cast<size_t>(M), 8));
  const void* Wp[2] = {W, W_up};
  const void* Ap[2] = {A, A_up};
  const void* Bp[2] = {B, B_up};
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };

  // 1. activation backward: dZ = dY * act'(Z) as hi + lo bf16
  const void* dZ[2] = {dY, nullptr};
  if (d->act != LORA_ACT_IDENTITY) {
    const long long n = static_cast<long long>(M) * d->d_out;
    const int grid = grid_for(n / 8, 256, dev.sms);
    if (swiglu) {
      act_bwd_kernel<true><<<grid, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(dY), Z_save, Z_save + static_cast<size_t>(M) * d->d_out, n,
          static_cast<__nv_bfloat16*>(at(L.dz_hi[0])), static_cast<__nv_bfloat16*>(at(L.dz_lo[0])),
          static_cast<__nv_bfloat16*>(at(L.dz_hi[1])), static_cast<__nv_bfloat16*>(at(L.dz_lo[1])));
    } else {
      act_bwd_kernel<false><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(dY), Z_save, nullptr, n,
                                                  static_cast<__nv_bfloat16*>(at(L.dz_hi[0])),
                                                  static_cast<__nv_bfloat16*>(at(L.dz_lo[0])), nullptr, nullptr);
    }
    LORA_TRY(check_launch("act_bwd_kernel"));
    for (int j = 0; j < np; ++j) dZ[j] = at(L.dz_hi[j]);
  }

  // 2. B^T and T (saved or recomputed) as s*T split into hi + lo, transposed
  if (r > 0) {
    for (int j = 0; j < np; ++j) {
      LORA_TRY(transpose_b(Bp[j], d->d_out, r, at(L.bt[j]), dev.sms, st));
      const float* Tj = T_save ? T_save + static_cast<size_t>(j) * M * r : nullptr;
      if (Tj == nullptr) {
        RankGemmParams q;
        std::memset(&q, 0, sizeof(q));
        bool ok = make_tm(&q.tm_a[0], X, d->d_in, M, d->d_in, 64, 128) &&
                  make_tm(&q.tm_b[0], Ap[j], d->d_in, r, d->d_in, 64, RP);
        if (!ok) return LORA_ERR_CUDA;
        q.rows = M;
        q.K = static_cast<int>(d->d_in);
        q.m_tiles = static_cast<int>(ceil_div(M, 128));
        q.kb_per_split = static_cast<int>(ceil_div(ceil_div(d->d_in, 64), L.splits_t));
        q.partial = static_cast<float*>(at(L.part_u));
        q.status = status;
        LORA_TRY(launch_rank_rp<false, 1>(RP, q, L.splits_t, st));
        LORA_TRY(reduce_partials(q.partial, L.splits_t, M, RP, r, nullptr, static_cast<float*>(at(L.tw[j])), 0,
                                 dev.sms, st));
        Tj = static_cast<const float*>(at(L.tw[j]));
      }
      LORA_TRY(rank_split_t(Tj, M, r, d->s, at(L.tt_hi[j]), at(L.tt_lo[j]), M8, dev.sms, st));
    }
  }

  // 3. dX = dZ W + s U A with U = dZ B (U saved for dA)
  {
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    bool ok = true;
    for (int j = 0; j < np; ++j) {
      ok = ok && make_tm(&p.tm_a[j], dZ[j], d->d_out, M, d->d_out, 64, 128);
      ok = ok && make_tm(&p.tm_w[j], Wp[j], d->d_in, d->d_out, d->d_in, 64, 64);
      if (r > 0) {
        ok = ok && make_tm(&p.tm_r[j], at(L.bt[j]), d->d_out, r, d->d_out, 64, RP);
        ok = ok && make_tm(&p.tm_up[j], Ap[j], d->d_in, r, d->d_in, 64, RP);
      }
    }
    if (!ok) return LORA_ERR_CUDA;
    p.M = M;
    p.N = static_cast<int>(d->d_in);
    p.K = static_cast<int>(d->d_out);
    p.r = r;
    p.s = d->s;
    p.out = static_cast<__nv_bfloat16*>(dX);
    p.rank_save = r > 0 ? static_cast<float*>(at(L.uw)) : nullptr;
    p.z_save = nullptr;
    p.status = status;
    p.m_tiles = static_cast<int>(ceil_div(M, kBM));
    p.n_tiles = static_cast<int>(ceil_div(d->d_in, 256));
    p.num_tiles = p.m_tiles * p.n_tiles;
    p.group_m = 8;
    if (swiglu) LORA_TRY((launch_gemm_rp<true, 2, kEpiGrad>(RP, p, dev.sms, st)));
    else LORA_TRY((launch_gemm_rp<true, 1, kEpiGrad>(RP, p, dev.sms, st)));
  }
  if (r == 0) return LORA_OK;

  for (int j = 0; j < np; ++j) {
    // U for pair j lives right after pair j-1's (the kernel saves [npair][M x r]).
    float* Uj = static_cast<float*>(at(L.uw)) + static_cast<size_t>(j) * M * r;
    // 4. act != identity: add the dZ_lo B part of U
    if (d->act != LORA_ACT_IDENTITY) {
      RankGemmParams q;
      std::memset(&q, 0, sizeof(q));
      bool ok = make_tm(&q.tm_a[0], at(L.dz_lo[j]), d->d_out, M, d->d_out, 64, 128) &&
                make_tm(&q.tm_b[0], at(L.bt[j]), d->d_out, r, d->d_out, 64, RP);
      if (!ok) return LORA_ERR_CUDA;
      q.rows = M;
      q.K = static_cast<int>(d->d_out);
      q.m_tiles = static_cast<int>(ceil_div(M, 128));
      q.kb_per_split = static_cast<int>(ceil_div(ceil_div(d->d_out, 64), L.splits_u));
      q.partial = static_cast<float*>(at(L.part_u));
      q.status = status;
      LORA_TRY(launch_rank_rp<false, 1>(RP, q, L.splits_u, st));
      LORA_TRY(reduce_partials(q.partial, L.splits_u, M, RP, r, Uj, Uj, 0, dev.sms, st));
    }
    // 5. s U as hi + lo, transposed
    LORA_TRY(rank_split_t(Uj, M, r, d->s, at(L.ut_hi[j]), at(L.ut_lo[j]), M8, dev.sms, st));
    // 6. dA^T = X^T (s U)
    {
      RankGemmParams q;
      std::memset(&q, 0, sizeof(q));
      bool ok = make_tm(&q.tm_a[0], X, d->d_in, M, d->d_in, 64, 64) &&
                make_tm(&q.tm_b[0], at(L.ut_hi[j]), M, r, M8, 64, RP) &&
                make_tm(&q.tm_b[1], at(L.ut_lo[j]), M, r, M8, 64, RP);
      if (!ok) return LORA_ERR_CUDA;
      q.rows = static_cast<int>(d->d_in);
      q.K = M;
      q.m_tiles = static_cast<int>(ceil_div(d->d_in, 128));
      q.kb_per_split = static_cast<int>(ceil_div(ceil_div(M, 64), L.splits_a));
      q.partial = static_cast<float*>(at(L.part_a));
      q.status = status;
      LORA_TRY(launch_rank_rp<true, 2>(RP, q, L.splits_a, st));
      LORA_TRY(reduce_partials(q.partial, L.splits_a, static_cast<int>(d->d_in), RP, r, nullptr, dAp[j], 1, dev.sms,
                               st));
    }
    // 7. dB = dZ^T (s T)
    {
      RankGemmParams q;
      std::memset(&q, 0, sizeof(q));
      bool ok = make_tm(&q.tm_a[0], dZ[j], d->d_out, M, d->d_out, 64, 64) &&
                make_tm(&q.tm_b[0], at(L.tt_hi[j]), M, r, M8, 64, RP) &&
                make_tm(&q.tm_b[1], at(L.tt_lo[j]), M, r, M8, 64, RP);
      if (d->act != LORA_ACT_IDENTITY) ok = ok && make_tm(&q.tm_a[1], at(L.dz_lo[j]), d->d_out, M, d->d_out, 64, 64);
      if (!ok) return LORA_ERR_CUDA;
      q.rows = static_cast<int>(d->d_out);
      q.K = M;
      q.m_tiles = static_cast<int>(ceil_div(d->d_out, 128));
      q.kb_per_split = static_cast<int>(ceil_div(ceil_div(M, 64), L.splits_b));
      q.partial = static_cast<float*>(at(L.part_b));
      q.status = status;
      if (d->act == LORA_ACT_IDENTITY) LORA_TRY((launch_rank_rp<true, 2>(RP, q, L.splits_b, st)));
      else LORA_TRY((launch_rank_rp<true, 3>(RP, q, L.splits_b, st)));
      LORA_TRY(reduce_partials(q.partial, L.splits_b, static_cast<int>(d->d_out), RP, r, nullptr, dBp[j], 0,
                               dev.sms, st));
    }
  }
  return LORA_OK;
}

}  // extern "C"
