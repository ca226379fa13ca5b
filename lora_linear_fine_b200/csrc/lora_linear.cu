// lora_linear.cu — the C ABI (include/lora_linear.h): argument checks, the
// workspace layout, tensor-map encoding and the launch sequence of the forward
// and backward of the fused LoRA-adapted linear layer on sm_100a.
#include "lora_linear.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <vector>
#include <map>
#include <mutex>
#include <tuple>

#include "lora_mma.cuh"
#include "lora_rank.cuh"
#include "lora_rank2d.cuh"
#include "lora_small_m.cuh"
#include "lora_w4.cuh"
#include "lora_dropout.cuh"
#include "lora_norm_rope.cuh"
#include "lora_ce.cuh"

namespace {

using namespace lora;

constexpr int kAbiVersion = 1;
constexpr int kTargetCtas = 148;   // SM count of a B200; sets split-K widths
// Workspace header, zero at rest: the status block (word 0 is the status
// word; words kTFlagWord0 .. kTFlagWord0 + kTFlagWords are the shared-T
// forward GEMM's exit count and flag bits, which that kernel sets and
// zeroes again within one launch).
constexpr size_t kHeaderBytes = 256;
constexpr int kTFlagWord0 = 8;
static_assert((kTFlagWord0 + 1 + kTFlagWords) * 4 <= kHeaderBytes, "header too small for the shared-T flags");

// ---------------------------------------------------------------------------
// debug logging (LORA_LINEAR_DEBUG=1)
// ---------------------------------------------------------------------------
int debug_level() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_DEBUG");
    v = (e && e[0] >= '1' && e[0] <= '9') ? e[0] - '0' : 0;
  }
  return v;
}
bool debug_on() { return debug_level() >= 1; }
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
             uint32_t box_inner, uint32_t box_outer, bool f16 = false,
             CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUresult r = g_encode(tm, dt, 2, const_cast<void*>(ptr), dims, strides, box,
                              es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) LORA_LOG("cuTensorMapEncodeTiled failed (%d): inner=%llu outer=%llu box=%ux%u", (int)r,
                                  (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
  return r == CUDA_SUCCESS;
}

// fp32 [outer x inner] row-major (rows row_elems elements apart), 128-byte
// swizzle: the target of the fp32 logits' TMA stores (box 32 x box_outer).
bool make_tm_f32(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_elems,
                 uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) LORA_LOG("cuTensorMapEncodeTiled (fp32) failed (%d): inner=%llu outer=%llu", (int)r,
                                  (unsigned long long)inner, (unsigned long long)outer);
  return r == CUDA_SUCCESS;
}

// 3D bf16 view [K blocks][rows][64] of a row-major [rows x 64 nkb] matrix
// (rows row_elems elements apart), 128-byte swizzle: box 64 x box_rows x
// box_kb lands in shared memory as box_kb consecutive [box_rows x 64] tiles.
bool make_tm3(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t nkb, uint64_t row_elems, uint32_t box_rows,
              uint32_t box_kb) {
  cuuint64_t dims[3] = {64, rows, nkb};
  cuuint64_t strides[2] = {row_elems * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_kb};
  cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) LORA_LOG("cuTensorMapEncodeTiled (3D) failed (%d): rows=%llu nkb=%llu box=%ux%u", (int)r,
                                  (unsigned long long)rows, (unsigned long long)nkb, box_rows, box_kb);
  return r == CUDA_SUCCESS;
}

// Tensor map over a plain row-major array without swizzle (the 4-bit weight's
// codes and scales): inner x outer elements of elem_bytes, rows row_bytes apart.
bool make_tm_plain(CUtensorMap* tm, const void* ptr, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = g_encode(tm, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) LORA_LOG("cuTensorMapEncodeTiled (plain) failed (%d): inner=%llu outer=%llu box=%ux%u", (int)r,
                                  (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// argument checks and sizes
// ---------------------------------------------------------------------------
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int rank_pad(int64_t r) { return r == 0 ? 0 : (r <= 16 ? 16 : (r <= 32 ? 32 : (r <= 64 ? 64 : 128))); }

lora_status_t check_desc(const lora_linear_desc* d) {
  if (d == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->M < 0 || d->d_in <= 0 || d->d_out <= 0 || d->r < 0) return LORA_ERR_INVALID_ARG;
  if (d->act < LORA_ACT_IDENTITY || d->act > LORA_ACT_SWIGLU) return LORA_ERR_INVALID_ARG;
  if (d->M > (int64_t(1) << 31) - 1 || d->d_in > (int64_t(1) << 30) || d->d_out > (int64_t(1) << 30))
    return LORA_ERR_UNSUPPORTED;
  if (d->d_in % 8 != 0 || d->d_out % 8 != 0) return LORA_ERR_ALIGNMENT;
  if (d->r % 8 != 0 || d->r > 128) return LORA_ERR_UNSUPPORTED;
  return LORA_OK;
}

// Workspace layouts (offsets in bytes, each 256-aligned, status word at 0).
struct Plan {
  int np = 1;              // projections: 2 for SwiGLU (gate, up)
  int RP = 0;              // r padded to the MMA granule (0, 16, 32, 64, 128)
  bool act_f16 = false;    // backward with an activation: fp16 dZ operands
  int64_t M8 = 8;
  // split-K widths of the rank passes (1 = results written directly)
  int splits_t = 1, splits_u = 1, splits_a = 1, splits_b = 1;
  // regions
  size_t s16[2] = {};                        // bf16 s*T (fwd) / s*U (bwd) [M x r]: LoRA K-block operand
  size_t t_ws = 0;                           // fp32 T [np][M x r] when the caller saves none (fwd)
  size_t bt[2] = {};                         // B^T [r x d_out] (bwd)
  size_t tt_hi[2] = {}, tt_lo[2] = {};       // (s*T)^T hi / lo [r x M8] (bwd, dB)
  size_t ut_hi[2] = {}, ut_lo[2] = {};       // (s*U)^T hi / lo [r x M8] (bwd, dA)
  size_t dz_hi[2] = {}, dz_lo[2] = {};     // activation backward: fp16 dZ operands
  // dX's N-side operands W and A are read in place, MN-major (with an
  // activation W as an fp16 copy).  A K-major copy of W paid for itself at
  // 16384 tokens while the epilogue stored its output per thread; with TMA
  // stores, reading W in place is faster at every size measured.
  size_t wt[2] = {};
  size_t part_t = 0, part_u = 0, part_a = 0, part_b = 0;   // split-K partials
  // backward rank passes on rank2d_kernel: U and dB from one read of dZ
  // (identity, r <= 32), dA over X
  bool dual = false;
  Rank2dSplit sp_dual, sp_a;
  // few-token forward
  bool small_m = false;
  int sm_nt = 16;                            // tokens padded to the MMA N granule
  size_t total = 0;
};

// The few-token forward applies to identity / SiLU with an adapter of rank at
// most 64 and at most kSmallMMax tokens.
bool small_m_applies(const lora_linear_desc* d) {
  return d->M > 0 && d->M <= kSmallMMax && d->r > 0 && d->r <= 64 && d->act != LORA_ACT_SWIGLU;
}

// Split-K width for a rank-r product with `tiles` row tiles and `nkb` 64-wide K blocks.
int rank_splits(int64_t tiles, int64_t nkb) {
  int64_t s = kTargetCtas / (tiles > 0 ? tiles : 1);
  if (s < 1) s = 1;
  if (s > nkb) s = nkb > 0 ? nkb : 1;
  if (s > 64) s = 64;
  return static_cast<int>(s);
}

// grad_f16: the backward's dZ comes as fp16 hi + lo even without an activation
// (the rotated projections: dZ = R^T dY), so it takes the activation's operand
// path: fp16 W copy, no K-major W^T, no fused U + dB pass.
Plan make_plan(const lora_linear_desc* d, bool backward, bool allow_small_m = true, bool grad_f16 = false) {
  Plan P;
  P.np = d->act == LORA_ACT_SWIGLU ? 2 : 1;
  P.RP = rank_pad(d->r);
  P.act_f16 = backward && (d->act != LORA_ACT_IDENTITY || grad_f16);
  P.M8 = static_cast<int64_t>(align_up(static_cast<size_t>(d->M > 0 ? d->M : 1), 8));
  const int64_t M = d->M, r = d->r;
  const int64_t tiles_m = ceil_div(M > 0 ? M : 1, 128);
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  auto partials = [&](int splits, int64_t tiles) -> size_t {
    return splits > 1 ? take(static_cast<size_t>(splits) * tiles * 128 * P.RP * 4) : 0;
  };
  if (!backward && allow_small_m && small_m_applies(d)) {
    // The few-token forward keeps everything on chip: no workspace regions.
    P.small_m = true;
    P.sm_nt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    P.total = off;
    return P;
  }
  if (r > 0) {
    // The LoRA branch rides the GEMM's K-loop as extra K-blocks fed by a rank
    // pass (T = X A^T, U = dZ B computed once per token): no rank columns in
    // tensor memory, which then holds two accumulator buffers.
    for (int j = 0; j < P.np; ++j) P.s16[j] = take(static_cast<size_t>(M) * r * 2);
    P.splits_t = rank_splits(tiles_m, ceil_div(d->d_in, 64));
    P.part_t = partials(P.splits_t, tiles_m);
    if (!backward) P.t_ws = take(static_cast<size_t>(P.np) * M * r * 4);
  }
  if (!backward) {
    P.total = off;
    return P;
  }
  for (int j = 0; j < P.np; ++j) {
    if (P.act_f16) P.wt[j] = take(static_cast<size_t>(d->d_out) * d->d_in * 2);
    if (P.act_f16) {
      P.dz_hi[j] = take(static_cast<size_t>(M) * d->d_out * 2);
      P.dz_lo[j] = take(static_cast<size_t>(M) * d->d_out * 2);
    }
  }
  if (r > 0) {
    for (int j = 0; j < P.np; ++j) {
      P.bt[j] = take(static_cast<size_t>(r) * d->d_out * 2);
      P.tt_hi[j] = take(static_cast<size_t>(r) * P.M8 * 2);
      P.tt_lo[j] = take(static_cast<size_t>(r) * P.M8 * 2);
      P.ut_hi[j] = take(static_cast<size_t>(r) * P.M8 * 2);
      P.ut_lo[j] = take(static_cast<size_t>(r) * P.M8 * 2);
    }
    const int64_t tiles_a = ceil_div(d->d_in, 128), tiles_b = ceil_div(d->d_out, 128);
    const int64_t nkb_tok = ceil_div(M > 0 ? M : 1, 64);
    // U and dB from one read of dY: identity, and r <= 64 (at r = 128 the
    // two accumulators and both B operands leave too little tensor and
    // shared memory)
    P.dual = !P.act_f16 && P.RP <= 64;
    if (P.dual) {
      P.sp_dual = rank2d_split(static_cast<int>(tiles_m), static_cast<int>(tiles_b), P.RP, true, true,
                               rank2d_max_rb(P.RP), kTargetCtas);
      if (P.sp_dual.fs > 1) P.part_u = take(static_cast<size_t>(P.sp_dual.fs) * tiles_m * 128 * P.RP * 4);
      if (P.sp_dual.ts > 1) P.part_b = take(static_cast<size_t>(P.sp_dual.ts) * tiles_b * 128 * P.RP * 4);
    } else {
      P.splits_u = rank_splits(tiles_m, ceil_div(d->d_out, 64));
      P.splits_b = rank_splits(tiles_b, nkb_tok);
      P.part_u = partials(P.splits_u, tiles_m);
      P.part_b = partials(P.splits_b, tiles_b);
    }
    P.sp_a = rank2d_split(static_cast<int>(tiles_m), static_cast<int>(tiles_a), P.RP, false, true, 0, kTargetCtas);
    if (P.sp_a.ts > 1) P.part_a = take(static_cast<size_t>(P.sp_a.ts) * tiles_a * 128 * P.RP * 4);
  }
  P.total = off;
  return P;
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

// Kernel launch with programmatic stream serialization: the kernel may start
// while its predecessor in the stream finishes (hiding launch latency and the
// prologue); every kernel of this library waits for its predecessor with
// griddepcontrol.wait before touching global memory.  LORA_LINEAR_PDL=0 turns
// the attribute off.  cluster2: launch as clusters of two CTAs.
bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_PDL");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool cluster2,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster2) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 2;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// benchmark instrumentation: CUDA events around the main GEMM launches
// ---------------------------------------------------------------------------
struct TimingState {
  bool enabled = false;
  std::vector<cudaEvent_t> ev[2];      // [direction] 2 events per launch
  size_t used[2] = {0, 0};
};
TimingState g_timing;
constexpr size_t kTimingPairs = 1024;

void timing_begin(int dir, cudaStream_t st) {
  if (!g_timing.enabled || g_timing.used[dir] >= kTimingPairs) return;
  cudaEventRecord(g_timing.ev[dir][2 * g_timing.used[dir]], st);
}

void timing_end(int dir, cudaStream_t st) {
  if (!g_timing.enabled || g_timing.used[dir] >= kTimingPairs) return;
  cudaEventRecord(g_timing.ev[dir][2 * g_timing.used[dir] + 1], st);
  ++g_timing.used[dir];
}

#define LORA_TRY(...)                           \
  do {                                          \
    const lora_status_t _s = (__VA_ARGS__);     \
    if (_s != LORA_OK) return _s;               \
  } while (0)

// ---------------------------------------------------------------------------
// kernel launchers
// ---------------------------------------------------------------------------
template <bool kAMN, int kRP, int kNA, int kNB, bool kF16>
lora_status_t launch_rank(const RankGemmParams& p, int splits, cudaStream_t st) {
  using C = RankCfg<kAMN, kRP, kNA, kNB, kF16>;
  auto k = rank_gemm_kernel<kAMN, kRP, kNA, kNB, kF16>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return cuda_error("cudaFuncSetAttribute(rank)");
  LORA_LOG("rank mn=%d RP=%d na=%d nb=%d f16=%d pairs=%d rows=%d K=%d tiles=%d splits=%d", (int)kAMN, kRP, kNA,
           kNB, (int)kF16, p.npairs, p.rows, p.K, p.m_tiles, splits);
  launch_k(k, dim3(p.m_tiles * splits), dim3(kRankThreads), C::kSmemBytes, st, false, p);
  return check_launch("rank_gemm_kernel");
}

template <bool kAMN, int kNA, int kNB, bool kF16>
lora_status_t launch_rank_rp(int RP, const RankGemmParams& p, int splits, cudaStream_t st) {
  switch (RP) {
    case 16: return launch_rank<kAMN, 16, kNA, kNB, kF16>(p, splits, st);
    case 32: return launch_rank<kAMN, 32, kNA, kNB, kF16>(p, splits, st);
    case 64: return launch_rank<kAMN, 64, kNA, kNB, kF16>(p, splits, st);
    case 128: return launch_rank<kAMN, 128, kNA, kNB, kF16>(p, splits, st);
    default: return LORA_ERR_UNSUPPORTED;
  }
}

int grid_for(long long n, int per_block, int sms) {
  long long g = (n + per_block - 1) / per_block;
  if (g > static_cast<long long>(sms) * 8) g = static_cast<long long>(sms) * 8;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// A rows x r rank product sum_q A[pa[q]] * B[pb[q]] over K (64-wide blocks
// split `splits` ways).  splits == 1: the kernel writes `out` directly;
// otherwise it writes fp32 partials to `partial` and reduce_rank finishes.
struct RankJob {
  bool a_mn = false;   // A read MN-major (result rows are the A tensor's columns)
  bool f16 = false;    // A and B operands are fp16 (else bf16)
  const void* a[2] = {nullptr, nullptr};
  int64_t a_inner = 0, a_outer = 0, a_ld = 0;     // A tensors share one shape
  const void* b[2] = {nullptr, nullptr};
  int64_t b_inner = 0, b_ld = 0;                  // B tensors: r rows x b_inner
  int na = 1, nb = 1, npairs = 1;
  int pa[4] = {0, 0, 0, 0}, pb[4] = {0, 0, 0, 0};
  int rows = 0, K = 0;
  float* partial = nullptr;
  int splits = 1;
  RankOut out = {};
  const uint8_t* mask = nullptr;   // dropout keep bits of the K-major A (X), [rows x mask_ld] bytes
  int mask_ld = 0;
};

RankOut rank_out(int rows, int r) {
  RankOut o;
  std::memset(&o, 0, sizeof(o));
  o.rows = rows;
  o.r = r;
  o.scale = 1.0f;
  return o;
}

lora_status_t run_rank_gemm(const RankJob& J, int RP, int r, uint32_t* status, cudaStream_t st) {
  RankGemmParams q;
  std::memset(&q, 0, sizeof(q));
  bool ok = true;
  const int ks = rank_ks(J.na, RP);   // 64-wide K blocks per stage (RankCfg::kKS)
  for (int i = 0; i < J.na; ++i)
    ok = ok && make_tm(&q.tm_a[i], J.a[i], J.a_inner, J.a_outer, J.a_ld, 64, J.a_mn ? 64 * ks : 128, J.f16);
  for (int i = 0; i < J.nb; ++i) ok = ok && make_tm(&q.tm_b[i], J.b[i], J.b_inner, r, J.b_ld, 64, RP, J.f16);
  if (!ok) return LORA_ERR_CUDA;
  q.rows = J.rows;
  q.K = J.K;
  q.m_tiles = static_cast<int>(ceil_div(J.rows, 128));
  q.kb_per_split = static_cast<int>(ceil_div(ceil_div(J.K, 64 * ks), J.splits));
  q.npairs = J.npairs;
  for (int i = 0; i < 4; ++i) { q.pa[i] = J.pa[i]; q.pb[i] = J.pb[i]; }
  q.partial = J.splits > 1 ? J.partial : nullptr;
  q.out = J.out;
  q.status = status;
  q.mask = J.mask;
  q.mask_ld = J.mask_ld;
  if (J.a_mn) {
    if (J.na == 1 && J.nb == 2 && !J.f16) return launch_rank_rp<true, 1, 2, false>(RP, q, J.splits, st);
    if (J.na == 2 && J.nb == 2 && J.f16) return launch_rank_rp<true, 2, 2, true>(RP, q, J.splits, st);
  } else {
    if (J.na == 1 && J.nb == 1 && !J.f16) return launch_rank_rp<false, 1, 1, false>(RP, q, J.splits, st);
    if (J.na == 2 && J.nb == 1 && J.f16) return launch_rank_rp<false, 2, 1, true>(RP, q, J.splits, st);
  }
  return LORA_ERR_UNSUPPORTED;
}

RankReduceJob reduce_job(const RankJob& J, int RP) {
  RankReduceJob R;
  R.partial = J.partial;
  R.splits = J.splits;
  R.rows_pad = static_cast<int>(ceil_div(J.rows, 128) * 128);
  R.RP = RP;
  R.out = J.out;
  return R;
}

// Fixed-order reduction of up to two split results in one launch.
lora_status_t launch_reduce(RankReduceJob* R, int n, cudaStream_t st) {
  if (n == 0) return LORA_OK;
  long long blocks = 0;
  for (int i = 0; i < n; ++i) {
    // rows per block: all kReduceRows while there are many rows, fewer (a
    // power of two) so that a short result still spreads over >= 256 blocks
    int rpb = kReduceRows;
    while (rpb > 1 && (R[i].out.rows + rpb - 1) / rpb < 256) rpb >>= 1;
    R[i].rpb = rpb;
    const long long b = (R[i].out.rows + rpb - 1) / rpb;
    blocks = b > blocks ? b : blocks;
  }
  if (n == 1) R[1] = R[0];
  long long gx = blocks;
  if (gx > 1184) gx = 1184;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(n), 1);
  launch_k(reduce_rank_kernel, grid, dim3(256), 0, st, false, R[0], R[1]);
  return check_launch("reduce_rank_kernel");
}

// Finish the jobs that were split (at most two, one launch).
lora_status_t finish_rank(const RankJob* j0, const RankJob* j1, int RP, cudaStream_t st) {
  const RankJob* js[2] = {j0, j1};
  RankReduceJob R[2];
  int n = 0;
  for (const RankJob* J : js) {
    if (J == nullptr || J->splits <= 1) continue;
    R[n++] = reduce_job(*J, RP);
  }
  return launch_reduce(R, n, st);
}

// One rank2d_kernel pass over Z [mtok x F] (bf16): the row product Z RB
// (rb = RB^T [r x F], or null) and/or the col product Z^T (CB_hi + CB_lo)
// (cb = [r x mtok] parts with row stride ld_cb), then the fixed-order
// reduction of whichever result was split.
template <int kRP, bool kRow, bool kCol>
lora_status_t launch_rank2d_t(const Rank2dParams& p, int grid, cudaStream_t st) {
  using C = Rank2dCfg<kRP, kRow, kCol>;
  auto k = rank2d_kernel<kRP, kRow, kCol>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return cuda_error("cudaFuncSetAttribute(rank2d)");
  LORA_LOG("rank2d RP=%d row=%d col=%d grid=%d a=%d b=%d fs=%d stages=%d", kRP, (int)kRow, (int)kCol, grid,
           p.a_tiles, p.b_blocks, p.fs, C::kStages);
  launch_k(k, dim3(grid), dim3(kRank2dThreads), C::kSmemBytes, st, false, p);
  return check_launch("rank2d_kernel");
}

template <bool kRow, bool kCol>
lora_status_t launch_rank2d_rp(int RP, const Rank2dParams& p, int grid, cudaStream_t st) {
  switch (RP) {
    case 16: return launch_rank2d_t<16, kRow, kCol>(p, grid, st);
    case 32: return launch_rank2d_t<32, kRow, kCol>(p, grid, st);
    case 64: return launch_rank2d_t<64, kRow, kCol>(p, grid, st);
    case 128:
      if constexpr (!kRow) return launch_rank2d_t<128, kRow, kCol>(p, grid, st);   // col product only
      else return LORA_ERR_UNSUPPORTED;
    default: return LORA_ERR_UNSUPPORTED;
  }
}

lora_status_t run_rank2d(const void* Z, int64_t F, int64_t mtok, int r, int RP, const void* rb, const void* cb_hi,
                         const void* cb_lo, int64_t ld_cb, const Rank2dSplit& sp, float* row_partial,
                         float* col_partial, const RankOut& row_out, const RankOut& col_out, uint32_t* status,
                         cudaStream_t st, const uint8_t* mask = nullptr) {
  const bool row = rb != nullptr, col = cb_hi != nullptr;
  Rank2dParams p;
  std::memset(&p, 0, sizeof(p));
  if (mask != nullptr && row) return LORA_ERR_UNSUPPORTED;   // masking serves the col-only pass over X
  p.mask = mask;
  p.mask_ld = static_cast<int>(F / 8);
  bool ok = make_tm(&p.tm_z, Z, F, mtok, F, 64, 128);
  if (row) ok = ok && make_tm(&p.tm_rb, rb, F, r, F, 64, RP);
  if (col) ok = ok && make_tm(&p.tm_cb[0], cb_hi, mtok, r, ld_cb, 64, RP) && make_tm(&p.tm_cb[1], cb_lo, mtok, r, ld_cb, 64, RP);
  if (!ok) return LORA_ERR_CUDA;
  p.mtok = static_cast<int>(mtok);
  p.F = static_cast<int>(F);
  p.m_tiles = static_cast<int>(ceil_div(mtok, 128));
  p.f_blocks = static_cast<int>(ceil_div(F, 128));
  p.a_tiles = sp.a;
  p.b_blocks = sp.b;
  p.fs = sp.fs;
  p.row_partial = sp.fs > 1 ? row_partial : nullptr;
  p.col_partial = sp.ts > 1 ? col_partial : nullptr;
  p.row_out = row_out;
  p.col_out = col_out;
  p.status = status;
  const int grid = sp.ts * sp.fs;
  lora_status_t rs;
  if (row && col) rs = launch_rank2d_rp<true, true>(RP, p, grid, st);
  else if (col) rs = launch_rank2d_rp<false, true>(RP, p, grid, st);
  else return LORA_ERR_UNSUPPORTED;
  LORA_TRY(rs);
  RankReduceJob R[2];
  int n = 0;
  if (row && sp.fs > 1) {
    R[n].partial = row_partial;
    R[n].splits = sp.fs;
    R[n].rows_pad = p.m_tiles * 128;
    R[n].RP = RP;
    R[n].out = row_out;
    ++n;
  }
  if (col && sp.ts > 1) {
    R[n].partial = col_partial;
    R[n].splits = sp.ts;
    R[n].rows_pad = p.f_blocks * 128;
    R[n].RP = RP;
    R[n].out = col_out;
    ++n;
  }
  return launch_reduce(R, n, st);
}

// T_j = X A_j^T written to `out` (split K finished in place).
// T_j = X A_j^T; with a dropout mask, T_j = (X * m) A_j^T with the mask applied
// to X's tiles inside the pass.
lora_status_t rank_T(const lora_linear_desc* d, const Plan& P, const void* X, const void* Aj, const RankOut& out,
                     uint8_t* ws, uint32_t* status, cudaStream_t st, const uint8_t* mask = nullptr) {
  RankJob J;
  J.a[0] = X;
  J.mask = mask;
  J.mask_ld = static_cast<int>(d->d_in / 8);
  J.a_inner = d->d_in;
  J.a_outer = d->M;
  J.a_ld = d->d_in;
  J.b[0] = Aj;
  J.b_inner = d->d_in;
  J.b_ld = d->d_in;
  J.rows = static_cast<int>(d->M);
  J.K = static_cast<int>(d->d_in);
  J.partial = reinterpret_cast<float*>(ws + P.part_t);
  J.splits = P.splits_t;
  J.out = out;
  LORA_TRY(run_rank_gemm(J, P.RP, static_cast<int>(d->r), status, st));
  return finish_rank(&J, nullptr, P.RP, st);
}

// ---------------------------------------------------------------------------
// the LoRA GEMM (lora_mma_kernel): launch as single CTAs or CTA pairs
// ---------------------------------------------------------------------------
bool pair_kernel_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_PAIR");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

// LORA_LINEAR_FUSED_T=0 turns off the forward GEMM's fused T, so that the
// separate T pass runs instead (for comparisons); LORA_LINEAR_SHARED_T=0
// turns off only its multi-tile form (a shared T per row block).
bool fused_t_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_FUSED_T");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}
bool shared_t_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("LORA_LINEAR_SHARED_T");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

template <bool kPair, bool kBwd, int kNPair, int kEpi>
lora_status_t launch_mma(const MmaParams& p0, int sms, cudaStream_t st) {
  using C = MmaCfg<kPair, kBwd, kNPair, kEpi>;
  auto k = lora_mma_kernel<kPair, kBwd, kNPair, kEpi>;
  MmaParams p = p0;
  if constexpr (C::kTmaOut) {
    // the epilogue's TMA stores: bf16 out [M x N], boxes of 64 columns x 32 rows
    if (p.out == nullptr || !make_tm(&p.tm_out, p.out, p.N, p.M, p.N, 64, 32)) return LORA_ERR_CUDA;
  }
  if constexpr (C::kTmaRope) {
    // the rotated output's TMA stores: bf16 out [M x N], boxes of 32 columns x 32 rows, 64-byte swizzle
    if (p.out == nullptr || !make_tm(&p.tm_out, p.out, p.N, p.M, p.N, 32, 32, false, CU_TENSOR_MAP_SWIZZLE_64B))
      return LORA_ERR_CUDA;
  }
  if constexpr (C::kTmaAct) {
    // the SiLU / SwiGLU forward's TMA stores: bf16 Y (boxes of 64 columns x
    // 32 rows) and, when saved, fp32 Z (32 x 32; SwiGLU: gate, then up)
    if (p.out == nullptr || !make_tm(&p.tm_out, p.out, p.N, p.M, p.N, 64, 32)) return LORA_ERR_CUDA;
    if (p.z_save != nullptr) {
      for (int j = 0; j < (C::kSwigluFwd ? 2 : 1); ++j)
        if (!make_tm_f32(&p.tm_z[j], p.z_save + static_cast<size_t>(j) * p.M * p.N, p.N, p.M, p.N, 32, 32))
          return LORA_ERR_CUDA;
    }
  }
  if constexpr (C::kTmaZ) {
    // the fp32 logits' TMA stores: out_f32 [M x N], boxes of 32 columns x 32 rows
    if (p.out_f32 == nullptr || !make_tm_f32(&p.tm_out, p.out_f32, p.N, p.M, p.N, 32, 32)) return LORA_ERR_CUDA;
  }
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return cuda_error("cudaFuncSetAttribute(mma)");
  const int max_units = kPair ? sms / 2 : sms;
  const int units = p.num_tiles < max_units ? p.num_tiles : max_units;
  LORA_LOG("mma pair=%d bwd=%d npair=%d epi=%d tiles=%d units=%d smem=%d stages=%d lora_ksteps=%d", (int)kPair,
           (int)kBwd, kNPair, kEpi, p.num_tiles, units, C::kSmemBytes, C::kStages, p.lora_ksteps);
  const cudaError_t e = launch_k(k, dim3(static_cast<unsigned>(units * C::kCtas)), dim3(kMmaThreads), C::kSmemBytes,
                                 st, kPair, p);
  if (e != cudaSuccess) {
    LORA_LOG("mma launch: %s", cudaGetErrorString(e));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return LORA_ERR_CUDA;
  }
  return check_launch("lora_mma_kernel");
}

// Raster choice for the GEMM: keep in L2 whichever operand fits.  m_bytes /
// n_bytes: total bytes of the M-side / N-side operands streamed by the K-loop.
void set_raster(MmaParams& p, bool pair, double m_bytes, double n_bytes) {
  constexpr double kL2Resident = 64.0 * 1024 * 1024;   // comfortably inside the 126 MB L2
  if (m_bytes <= kL2Resident && n_bytes > m_bytes) {
    p.group_along_n = 1;   // sweep all M tiles per group of N tiles: the N side streams once
    p.group = 1;
  } else {
    p.group_along_n = 0;   // sweep all N tiles per group of M tiles: the N side stays in L2
    p.group = pair ? 4 : 8;
  }
}

template <bool kBwd, int kNPair, int kEpi>
lora_status_t launch_mma_any(bool pair, const MmaParams& p, int sms, cudaStream_t st) {
  return pair ? launch_mma<true, kBwd, kNPair, kEpi>(p, sms, st) : launch_mma<false, kBwd, kNPair, kEpi>(p, sms, st);
}

// Failure-detection self-test: one thread waits, through the library's
// bounded mbarrier wait, for a phase that nothing completes.  The wait gives
// up after `limit` cycles and ORs kStatusWaitTimeout into the status word.
__global__ void selftest_wait_kernel(uint32_t* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ uint32_t flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    AbortCtl ctl{&flag, status};
    mbar_wait(&bar, 0u, ctl, limit);
  }
}

lora_status_t common_checks(const lora_linear_desc* d, void* ws, size_t ws_bytes, size_t need, DevInfo* dev) {
  LORA_TRY(check_desc(d));
  LORA_TRY(device_info(dev));
  if (dev->major != 10 || dev->minor != 0) return LORA_ERR_ARCH;
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return LORA_ERR_WORKSPACE;
  return LORA_OK;
}

// Few tokens: bound by reading W once; one cluster per 128-row slice of W.
// W is bf16, or (Wq != null) the 4-bit codes Wq with scales Ws.
lora_status_t run_small_m_fwd(const lora_linear_desc* d, int nt, const void* X, const void* W, const void* Wq,
                              const void* Ws, const void* A, const void* B, void* Y, float* T_save, float* Z_save,
                              uint32_t* status, cudaStream_t st, const void* Wt = nullptr) {
  const int64_t M = d->M, r = d->r;
  SmallMParams q;
  std::memset(&q, 0, sizeof(q));
  const bool w4 = Wq != nullptr || Wt != nullptr;
  const uint32_t kps = static_cast<uint32_t>(small_m_kps(nt, w4, small_m_ar(r)));
  q.Wt = static_cast<const uint8_t*>(Wt);
  bool ok = Wt != nullptr ? make_tm_plain(&q.tm_ws, Ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->d_out,
                                          d->d_in / kW4Group, d->d_out * 2, 128, kps)
          : w4 ? make_tm_plain(&q.tm_w, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, d->d_in / 2, d->d_out, d->d_in / 2, 32,
                               128) &&
                     make_tm_plain(&q.tm_ws, Ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d->d_out, d->d_in / kW4Group,
                                   d->d_out * 2, 128, kps)
               : make_tm(&q.tm_w, W, d->d_in, d->d_out, d->d_in, 64, 128);
  if (!ok ||
      !make_tm(&q.tm_a, A, d->d_in, r, d->d_in, 64, static_cast<uint32_t>(align_up(static_cast<size_t>(r), 16))) ||
      !make_tm(&q.tm_x, X, d->d_in, M, d->d_in, 64, static_cast<uint32_t>(nt)))
    return LORA_ERR_CUDA;
  q.B = static_cast<const __nv_bfloat16*>(B);
  q.Y = static_cast<__nv_bfloat16*>(Y);
  q.T_save = T_save;
  q.Z_save = d->act == LORA_ACT_SILU ? Z_save : nullptr;
  q.status = status;
  q.M = static_cast<int>(M);
  q.d_in = static_cast<int>(d->d_in);
  q.d_out = static_cast<int>(d->d_out);
  q.r = static_cast<int>(r);
  q.s = d->s;
  q.act = d->act;
  q.a_rows = static_cast<int>(align_up(static_cast<size_t>(r), 16));
  // One TMA load per operand and stage through 3D views when the K blocks
  // are whole (a 3D view cannot zero-fill a ragged last block); otherwise
  // one 2D box per K block into the same layout.
  if (d->d_in % 64 == 0) {
    const uint64_t nkb = static_cast<uint64_t>(d->d_in / 64);
    q.load3d = make_tm3(&q.tm_x3, X, M, nkb, d->d_in, static_cast<uint32_t>(nt), kps) &&
               make_tm3(&q.tm_a3, A, r, nkb, d->d_in, static_cast<uint32_t>(small_m_ar(r)), kps) &&
               (w4 || make_tm3(&q.tm_w3, W, d->d_out, nkb, d->d_in, 128, kps));
  }
  const int slices = static_cast<int>(ceil_div(d->d_out, 128));
  {
    // The cluster size depends only on the device and the shape: ask the
    // occupancy API once per (device, nt, w4, d_in, d_out) and keep the answer.
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int64_t, int64_t>, int> cache;
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    const auto key = std::make_tuple(dev_id, nt, static_cast<int>(w4) + 2 * small_m_ar(r), d->d_in, d->d_out);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it == cache.end()) it = cache.emplace(key, small_m_splits(nt, w4, r, d->d_in, d->d_out)).first;
    q.splits = it->second;
  }
  q.kb_per = static_cast<int>(ceil_div(ceil_div(d->d_in, 64), q.splits));
  const int grid = slices * q.splits;
  LORA_LOG("small_m M=%d nt=%d w4=%d slices=%d splits=%d kb_per=%d grid=%d", (int)M, nt, (int)w4, slices,
           q.splits, q.kb_per, grid);
  // LORA_LINEAR_DEBUG=2: per-CTA phase stamps, printed after the launch
  // (synchronises the stream; for debugging only).
  static unsigned long long* trace = nullptr;
  if (debug_level() >= 2 && trace == nullptr &&
      cudaMalloc(&trace, sizeof(unsigned long long) * 1024 * kSmTraceStride) != cudaSuccess)
    trace = nullptr;
  if (debug_level() >= 2 && trace != nullptr && grid <= 1024) {
    q.trace = trace;
    cudaMemsetAsync(trace, 0, sizeof(unsigned long long) * grid * kSmTraceStride, st);
  }
  const cudaError_t e = launch_small_m(q, nt, w4, slices, pdl_enabled(), st);
  if (e != cudaSuccess) {
    LORA_LOG("small_m launch: %s", cudaGetErrorString(e));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return LORA_ERR_CUDA;
  }
  const lora_status_t ls = check_launch("small_m_kernel");
  if (q.trace != nullptr && cudaStreamSynchronize(st) == cudaSuccess) {
    std::vector<unsigned long long> h(static_cast<size_t>(grid) * kSmTraceStride);
    cudaMemcpy(h.data(), trace, h.size() * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
    unsigned long long t0 = ~0ull;
    for (int b = 0; b < grid; ++b)
      t0 = h[b * kSmTraceStride] && h[b * kSmTraceStride] < t0 ? h[b * kSmTraceStride] : t0;
    static const char* names[kSmTracePoints] = {"entry", "first_issue", "first_data", "last_mma", "published",
                                                "synced", "t_summed", "combined", "exit", "dq_wait", "dq_work"};
    auto stats = [&](int k, const char* name) {
      double mn = 1e30, mx = 0, sum = 0;
      int n = 0;
      for (int b = 0; b < grid; ++b) {
        const unsigned long long v = h[b * kSmTraceStride + k];
        if (v == 0) continue;
        const double us = (v - t0) * 1e-3;
        mn = us < mn ? us : mn;
        mx = us > mx ? us : mx;
        sum += us;
        ++n;
      }
      if (n) LORA_LOG("small_m trace %-12s n=%3d min %7.2f mean %7.2f max %7.2f us", name, n, mn, sum / n, mx);
    };
    for (int k = 0; k < kSmTracePoints; ++k) {
      if (k == kTrDqWait || k == kTrDqWork) {   // durations, not stamps
        double tot = 0;
        int cnt = 0;
        for (int b = 0; b < grid; ++b)
          if (h[b * kSmTraceStride + k]) { tot += h[b * kSmTraceStride + k] * 1e-3; ++cnt; }
        if (cnt) LORA_LOG("small_m trace %-12s n=%3d mean total %7.2f us", names[k], cnt, tot / cnt);
        continue;
      }
      stats(k, names[k]);
    }
    char nm[32];
    for (int i = 0; i < kSmTraceStages; ++i) {
      std::snprintf(nm, sizeof nm, "issue[%d]", i);
      stats(kSmTracePoints + i, nm);
      std::snprintf(nm, sizeof nm, "full[%d]", i);
      stats(kSmTracePoints + kSmTraceStages + i, nm);
    }
  }
  return ls;
}

// 4-bit frozen base weight: shared checks and the expansion to bf16.
// Checks shared by the 4-bit entry points: the codes and scales of W (and of
// W_up for SwiGLU) are required and 16-byte aligned; d_in is a multiple of 64.
lora_status_t check_w4(const lora_linear_desc* d, const void* Wq, const void* Ws, const void* Wq_up,
                       const void* Ws_up) {
  LORA_TRY(check_desc(d));
  if (Wq == nullptr || Ws == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->act == LORA_ACT_SWIGLU && (Wq_up == nullptr || Ws_up == nullptr)) return LORA_ERR_INVALID_ARG;
  if (d->d_in % kW4Group != 0) return LORA_ERR_ALIGNMENT;
  const void* ptrs[] = {Wq, Ws, Wq_up, Ws_up};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

// Bytes of the bf16 weight(s) the tiled path expands into (after the regular
// workspace), 0 for the few-token forward, which reads the codes directly.
size_t w4_expand_bytes(const lora_linear_desc* d, bool backward) {
  if (!backward && small_m_applies(d)) return 0;
  const size_t np = d->act == LORA_ACT_SWIGLU ? 2 : 1;
  return np * static_cast<size_t>(d->d_out) * static_cast<size_t>(d->d_in) * 2;
}

lora_status_t dequant_w4(const void* Wq, const void* Ws, int64_t d_out, int64_t d_in, void* W, cudaStream_t st) {
  DevInfo dev;
  LORA_TRY(device_info(&dev));
  const long long n = d_out * (d_in / 16);
  launch_k(dequant_w4_kernel, dim3(grid_for(n, 256, dev.sms)), dim3(256), 0, st, false,
           static_cast<const uint8_t*>(Wq), static_cast<const __nv_bfloat16*>(Ws), static_cast<long long>(d_out),
           static_cast<int>(d_in), static_cast<__nv_bfloat16*>(W));
  return check_launch("dequant_w4_kernel");
}

// Dropout on the adapter branch's input: checks and workspace.
lora_status_t check_dropout(const lora_linear_desc* d, const void* X, const void* mask, const void* mask_up,
                            float p_drop) {
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return LORA_ERR_INVALID_ARG;
  if (d->M > 0 && (X == nullptr || mask == nullptr || (d->act == LORA_ACT_SWIGLU && mask_up == nullptr)))
    return LORA_ERR_INVALID_ARG;
  if (X != nullptr && !aligned16(X)) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

// The workspace of the layer without the few-token path (dropout always runs tiled).
size_t dropout_base_bytes(const lora_linear_desc* d, bool backward) {
  const size_t fwd = make_plan(d, false, false).total;
  if (!backward) return fwd;
  const size_t bwd = make_plan(d, true).total;
  return bwd > fwd ? bwd : fwd;
}

// Rotary tables of the attention-input projections: checks shared by the
// forward and the backward.
lora_status_t check_rope(const lora_linear_desc* d, const lora_rope_desc* rd, RopeTables* out) {
  if (rd == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->act != LORA_ACT_IDENTITY) return LORA_ERR_UNSUPPORTED;
  if (rd->head_dim != 64 && rd->head_dim != 128) return LORA_ERR_UNSUPPORTED;
  if (d->d_out % rd->head_dim != 0) return LORA_ERR_INVALID_ARG;
  if (rd->n_pos < 1 || rd->n_pos > (int64_t(1) << 31)) return LORA_ERR_INVALID_ARG;
  if (d->M > 0 && (rd->pos == nullptr || rd->cos == nullptr || rd->sin == nullptr)) return LORA_ERR_INVALID_ARG;
  if ((rd->cos != nullptr && !aligned16(rd->cos)) || (rd->sin != nullptr && !aligned16(rd->sin)) ||
      (reinterpret_cast<uintptr_t>(rd->pos) & 3u) != 0)
    return LORA_ERR_ALIGNMENT;
  out->pos = rd->pos;
  out->cos = rd->cos;
  out->sin = rd->sin;
  out->n_pos = rd->n_pos;
  out->half = rd->head_dim / 2;
  return LORA_OK;
}

lora_status_t check_arch(DevInfo* dev) {
  LORA_TRY(device_info(dev));
  return (dev->major == 10 && dev->minor == 0) ? LORA_OK : LORA_ERR_ARCH;
}

int norm_grid(int64_t M, const DevInfo& dev) {
  const int64_t blocks = ceil_div(M, kNormWarps);
  const int64_t cap = static_cast<int64_t>(dev.sms) * 8;   // 8 CTAs of 8 warps fill an SM
  return static_cast<int>(blocks < cap ? blocks : cap);
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

int lora_linear_abi_version(void) { return kAbiVersion; }

uint64_t lora_linear_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

lora_status_t lora_linear_timing_enable(int enable) {
  if (enable) {
    for (int dir = 0; dir < 2; ++dir) {
      while (g_timing.ev[dir].size() < 2 * kTimingPairs) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return cuda_error("cudaEventCreate");
        g_timing.ev[dir].push_back(e);
      }
      g_timing.used[dir] = 0;
    }
  }
  g_timing.enabled = enable != 0;
  return LORA_OK;
}

lora_status_t lora_linear_timing_read(double* fwd_ms, uint64_t* fwd_launches, double* bwd_ms,
                                      uint64_t* bwd_launches) {
  double ms[2] = {0.0, 0.0};
  for (int dir = 0; dir < 2; ++dir) {
    for (size_t i = 0; i < g_timing.used[dir]; ++i) {
      float t = 0.0f;
      if (cudaEventSynchronize(g_timing.ev[dir][2 * i + 1]) != cudaSuccess ||
          cudaEventElapsedTime(&t, g_timing.ev[dir][2 * i], g_timing.ev[dir][2 * i + 1]) != cudaSuccess)
        return cuda_error("cudaEventElapsedTime");
      ms[dir] += t;
    }
  }
  if (fwd_ms) *fwd_ms = ms[0];
  if (bwd_ms) *bwd_ms = ms[1];
  if (fwd_launches) *fwd_launches = g_timing.used[0];
  if (bwd_launches) *bwd_launches = g_timing.used[1];
  g_timing.used[0] = g_timing.used[1] = 0;
  return LORA_OK;
}

lora_status_t lora_linear_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_log2,
                                                void* stream) {
  if (workspace == nullptr || workspace_bytes < kHeaderBytes || !aligned16(workspace)) return LORA_ERR_WORKSPACE;
  if (limit_log2 < 10 || limit_log2 > 30) return LORA_ERR_INVALID_ARG;
  DevInfo dev;
  LORA_TRY(device_info(&dev));
  if (dev.major != 10 || dev.minor != 0) return LORA_ERR_ARCH;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace),
                                                                        1ll << limit_log2);
  return check_launch("selftest_wait_kernel");
}

const char* lora_status_string(lora_status_t s) {
  switch (s) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARG: return "invalid argument";
    case LORA_ERR_ALIGNMENT: return "misaligned pointer or dimension (16-byte pointers, d_in/d_out multiples of 8)";
    case LORA_ERR_UNSUPPORTED: return "unsupported shape or option (r must be 0 or a multiple of 8 up to 128)";
    case LORA_ERR_ARCH: return "current device is not sm_100 (B200)";
    case LORA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_DEVICE_STATUS: return "device status word is non-zero";
  }
  return "unknown status";
}

size_t lora_linear_workspace_size(const lora_linear_desc* desc, int for_backward) {
  if (check_desc(desc) != LORA_OK) return 0;
  const size_t fwd = make_plan(desc, false).total;
  if (for_backward == 0) return fwd;
  const size_t bwd = make_plan(desc, true).total;
  return bwd > fwd ? bwd : fwd;     // one workspace sized for the backward serves both
}

lora_status_t lora_linear_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || workspace_bytes < kHeaderBytes) return LORA_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
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

// The forward.  Xl[j] is the input of projection j's adapter branch (X; with
// dropout, fmasks[j] are the keep bits the T pass applies to its X tiles);
// allow_small_m = false keeps the tiled path for few tokens.
// Host-side argument checks of a forward (desc, required pointers,
// alignment): everything that needs neither the device nor the workspace.
static lora_status_t fwd_check_args(const lora_linear_desc* d, const void* X, const void* W, const void* A,
                                    const void* B, const void* W_up, const void* A_up, const void* B_up,
                                    const void* Y, const void* T_save, const void* Z_save) {
  LORA_TRY(check_desc(d));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  // with M == 0 the per-token tensors are empty and may be NULL
  if (W == nullptr || (d->M > 0 && (X == nullptr || Y == nullptr))) return LORA_ERR_INVALID_ARG;
  if (d->r > 0 && (A == nullptr || B == nullptr)) return LORA_ERR_INVALID_ARG;
  if (swiglu && (W_up == nullptr || (d->r > 0 && (A_up == nullptr || B_up == nullptr)))) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

static lora_status_t fwd_core(const lora_linear_desc* d, const void* X, const void* W, const void* A,
                              const void* B, const void* W_up, const void* A_up, const void* B_up, void* Y,
                              float* T_save, float* Z_save, void* workspace, size_t workspace_bytes, void* stream,
                              const void* const Xl[2], bool allow_small_m, const RopeTables* rope = nullptr,
                              const uint8_t* const fmasks[2] = nullptr) {
  LORA_TRY(fwd_check_args(d, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  const Plan P = make_plan(d, false, allow_small_m);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, P.total, &dev));
  if (d->M == 0) return LORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const int np = P.np, RP = P.RP;
  const int64_t M = d->M, r = d->r;

  if (P.small_m) return run_small_m_fwd(d, P.sm_nt, X, W, nullptr, nullptr, A, B, Y, T_save, Z_save, status, st);

  const void* Wp[2] = {W, W_up};
  const void* Ap[2] = {A, A_up};
  const void* Bp[2] = {B, B_up};
  const bool pair = pair_kernel_enabled() && M > 128;
  // T accumulated inside the forward GEMM (one identity projection, rotated
  // or not, r <= 64, no dropout), so that the separate T pass (and its
  // split-K reduction) is skipped and X is streamed by the GEMM alone:
  // - one GEMM tile per unit (a single wave, e.g. about a thousand tokens):
  //   every tile accumulates T in the free second accumulator buffer;
  // - at most one row block per unit (up to 256 x 74 tokens): the N-tile-0
  //   tile of each row block goes first on its unit, accumulates T there and
  //   publishes bf16(s T); the row block's other tiles load it for their
  //   LoRA block.
  const int64_t m_tiles1 = ceil_div(M, pair ? 256 : 128);
  const int64_t tiles1 = m_tiles1 * ceil_div(d->d_out, 256);
  const int64_t units1 = pair ? dev.sms / 2 : dev.sms;
  const bool t_in_gemm = fused_t_enabled() && r > 0 && RP <= 64 && np == 1 && d->act == LORA_ACT_IDENTITY &&
                         fmasks == nullptr;
  const bool share_t = t_in_gemm && tiles1 > units1 && m_tiles1 <= units1 && shared_t_enabled();
  const bool fuse_t = t_in_gemm && (tiles1 <= units1 || share_t);
  // 1. T_j = X A_j^T (fp32, saved for the backward) and bf16(s T_j) for the LoRA K-block
  if (r > 0 && !fuse_t) {
    for (int j = 0; j < np; ++j) {
      RankOut o = rank_out(static_cast<int>(M), static_cast<int>(r));
      o.f32 = T_save ? T_save + static_cast<size_t>(j) * M * r
                     : reinterpret_cast<float*>(ws + P.t_ws) + static_cast<size_t>(j) * M * r;
      o.s16 = reinterpret_cast<__nv_bfloat16*>(ws + P.s16[j]);
      o.scale = d->s;
      LORA_TRY(rank_T(d, P, Xl[j], Ap[j], o, ws, status, st, fmasks != nullptr ? fmasks[j] : nullptr));
    }
  }
  // 2. Z = [X | sT] [W | B]^T, activation, bf16 Y
  MmaParams p;
  std::memset(&p, 0, sizeof(p));
  const int outc = swiglu ? 128 : 256;
  const int brows = swiglu ? (pair ? 64 : 128) : (pair ? 128 : 256);   // N-side rows per CTA box
  bool ok = make_tm(&p.tm_a[0], X, d->d_in, M, d->d_in, 64, 128);
  for (int j = 0; j < np; ++j) {
    ok = ok && make_tm(&p.tm_w[j], Wp[j], d->d_in, d->d_out, d->d_in, 64, swiglu ? 128 : brows);
    if (r > 0) {
      ok = ok && make_tm(&p.tm_la[j], ws + P.s16[j], r, M, r, 64, 128);
      ok = ok && make_tm(&p.tm_lb[j], Bp[j], r, d->d_out, r, 64, brows);
    }
  }
  if (!ok) return LORA_ERR_CUDA;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(d->d_out);
  p.K = static_cast<int>(d->d_in);
  p.lora_ksteps = static_cast<int>((r + 15) / 16);
  p.out = static_cast<__nv_bfloat16*>(Y);
  p.z_save = d->act != LORA_ACT_IDENTITY ? Z_save : nullptr;
  p.status = status;
  p.m_tiles = static_cast<int>(ceil_div(M, pair ? 256 : 128));
  p.n_tiles = static_cast<int>(ceil_div(d->d_out, outc));
  p.num_tiles = p.m_tiles * p.n_tiles;
  set_raster(p, pair, 2.0 * M * d->d_in, 2.0 * np * d->d_out * d->d_in);
  timing_begin(0, st);
  lora_status_t rs;
  if (fuse_t) {
    p.am_rows = RP / (pair ? 2 : 1);
    p.rp = RP;
    p.r = static_cast<int>(r);
    p.lora_scale = d->s;
    p.t_save = T_save;
    if (share_t) {
      p.t_shared = 1;
      p.st_out = reinterpret_cast<__nv_bfloat16*>(ws + P.s16[0]);
      p.t_flags = status + kTFlagWord0;
    }
    if (!make_tm(&p.tm_am, A, d->d_in, r, d->d_in, 64, p.am_rows)) return LORA_ERR_CUDA;
    if (rope != nullptr) {
      p.rope = *rope;
      rs = launch_mma_any<false, 1, kMEpiRopeT>(pair, p, dev.sms, st);
    } else {
      rs = launch_mma_any<false, 1, kMEpiIdentityT>(pair, p, dev.sms, st);
    }
    timing_end(0, st);
    return rs;
  }
  if (rope != nullptr) {
    p.rope = *rope;
    rs = launch_mma_any<false, 1, kMEpiRope>(pair, p, dev.sms, st);
    timing_end(0, st);
    return rs;
  }
  switch (d->act) {
    case LORA_ACT_IDENTITY: rs = launch_mma_any<false, 1, kMEpiIdentity>(pair, p, dev.sms, st); break;
    case LORA_ACT_SILU: rs = launch_mma_any<false, 1, kMEpiSilu>(pair, p, dev.sms, st); break;
    default: rs = launch_mma_any<false, 2, kMEpiSwiglu>(pair, p, dev.sms, st); break;
  }
  timing_end(0, st);
  return rs;
}

lora_status_t lora_linear_fwd(const lora_linear_desc* d, const void* X, const void* W, const void* A, const void* B,
                              const void* W_up, const void* A_up, const void* B_up, void* Y, float* T_save,
                              float* Z_save, void* workspace, size_t workspace_bytes, void* stream) {
  const void* Xl[2] = {X, X};
  return fwd_core(d, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, workspace, workspace_bytes, stream, Xl, true);
}

// The backward.  Xl[j] is the input of projection j's adapter branch; with
// dropout masks (masks[0] != null) the rank passes mask their X tiles, and the
// dX GEMM forms the masked LoRA term in its accumulator before the main
// K-blocks (one projection) or runs without its LoRA K-blocks while
// dx_dropout_kernel adds the masked terms afterwards (SwiGLU).
static lora_status_t bwd_core(const lora_linear_desc* d, const void* dY, const void* X, const void* W, const void* A,
                              const void* B, const void* W_up, const void* A_up, const void* B_up,
                              const float* T_save, const float* Z_save, void* dX, float* dA, float* dB,
                              float* dA_up, float* dB_up, void* workspace, size_t workspace_bytes, void* stream,
                              const void* const Xl[2], const uint8_t* const masks[2],
                              const RopeTables* rope = nullptr, float* dXf = nullptr, int dXf_acc = 0) {
  LORA_TRY(check_desc(d));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  // with M == 0 the per-token tensors are empty and may be NULL; dXf (fp32,
  // written or added to) replaces the bf16 dX
  if (W == nullptr || (d->M > 0 && (dY == nullptr || X == nullptr || (dX == nullptr && dXf == nullptr))))
    return LORA_ERR_INVALID_ARG;
  if (d->r > 0 && (A == nullptr || B == nullptr || dA == nullptr || dB == nullptr)) return LORA_ERR_INVALID_ARG;
  if (swiglu && (W_up == nullptr || (d->r > 0 && (A_up == nullptr || B_up == nullptr || dA_up == nullptr ||
                                                  dB_up == nullptr))))
    return LORA_ERR_INVALID_ARG;
  if (d->act != LORA_ACT_IDENTITY && d->M > 0 && Z_save == nullptr) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up, dXf};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  const Plan P = make_plan(d, true, true, rope != nullptr);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, P.total, &dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int np = P.np, RP = P.RP;
  (void)RP;
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
  const int M = static_cast<int>(d->M);
  const int r = static_cast<int>(d->r);
  const int M8 = static_cast<int>(P.M8);
  const bool f16 = P.act_f16;
  const void* Wp[2] = {W, W_up};
  const void* Ap[2] = {A, A_up};
  const void* Bp[2] = {B, B_up};
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };

  // 1. dZ operands.  identity: dZ = dY (bf16, exact).  Otherwise dZ = dY * act'(Z)
  //    as fp16 hi + lo.  W for the dX product is read in place (an fp16 copy
  //    with an activation).
  const void* dZ[2] = {dY, nullptr};
  const void* dZlo[2] = {nullptr, nullptr};
  const void* Wmain[2] = {W, W_up};
  if (f16) {
    const long long n = static_cast<long long>(M) * d->d_out;
    const int grid = grid_for(n / 8, 256, dev.sms);
    if (rope != nullptr)
      launch_k(rope_bwd_kernel, dim3(grid_for(n / 16, 256, dev.sms)), dim3(256), 0, st, false,
               static_cast<const __nv_bfloat16*>(dY), *rope, static_cast<long long>(M), static_cast<int>(d->d_out),
               static_cast<__half*>(at(P.dz_hi[0])), static_cast<__half*>(at(P.dz_lo[0])), status);
    else if (swiglu)
      launch_k(act_bwd_kernel<true>, dim3(grid), dim3(256), 0, st, false, static_cast<const __nv_bfloat16*>(dY),
               static_cast<const float*>(Z_save), static_cast<const float*>(Z_save + static_cast<size_t>(M) * d->d_out),
               static_cast<long long>(n), static_cast<__half*>(at(P.dz_hi[0])), static_cast<__half*>(at(P.dz_lo[0])),
               static_cast<__half*>(at(P.dz_hi[1])), static_cast<__half*>(at(P.dz_lo[1])), status);
    else
      launch_k(act_bwd_kernel<false>, dim3(grid), dim3(256), 0, st, false, static_cast<const __nv_bfloat16*>(dY),
               static_cast<const float*>(Z_save), static_cast<const float*>(nullptr), static_cast<long long>(n),
               static_cast<__half*>(at(P.dz_hi[0])), static_cast<__half*>(at(P.dz_lo[0])),
               static_cast<__half*>(nullptr), static_cast<__half*>(nullptr), status);
    LORA_TRY(check_launch(rope != nullptr ? "rope_bwd_kernel" : "act_bwd_kernel"));
    const long long nw = static_cast<long long>(d->d_out) * d->d_in;
    for (int j = 0; j < np; ++j) {
      dZ[j] = at(P.dz_hi[j]);
      dZlo[j] = at(P.dz_lo[j]);
      launch_k(convert_f16_kernel, dim3(grid_for(nw / 8, 256, dev.sms)), dim3(256), 0, st, false,
               static_cast<const __nv_bfloat16*>(Wp[j]), static_cast<__half*>(at(P.wt[j])), static_cast<long long>(nw),
               status);
      LORA_TRY(check_launch("convert_f16_kernel"));
      Wmain[j] = at(P.wt[j]);
    }
  }

  // 2. B^T and (s T)^T hi/lo (from the saved T, or a rank pass recomputing
  //    T), in the dZ operand type.
  if (r > 0) {
    for (int j = 0; j < np; ++j) {
      const float* Tj = T_save ? T_save + static_cast<size_t>(j) * M * r : nullptr;
      // one thread per row and 8-column chunk
      const long long n = (d->d_out + (Tj ? M : 0)) * (r / 8);
      if (f16)
        launch_k(bwd_prep_kernel<__half>, dim3(grid_for(n, 256, dev.sms)), dim3(256), 0, st, false,
                 static_cast<const __nv_bfloat16*>(Bp[j]), static_cast<int>(d->d_out), r,
                 static_cast<__half*>(at(P.bt[j])), Tj, M, d->s,
                 static_cast<__half*>(at(P.tt_hi[j])), static_cast<__half*>(at(P.tt_lo[j])), M8, status);
      else
        launch_k(bwd_prep_kernel<__nv_bfloat16>, dim3(grid_for(n, 256, dev.sms)), dim3(256), 0, st, false,
                 static_cast<const __nv_bfloat16*>(Bp[j]), static_cast<int>(d->d_out), r,
                 static_cast<__nv_bfloat16*>(at(P.bt[j])), Tj, M, d->s,
                 static_cast<__nv_bfloat16*>(at(P.tt_hi[j])), static_cast<__nv_bfloat16*>(at(P.tt_lo[j])), M8,
                 status);
      LORA_TRY(check_launch("bwd_prep_kernel"));
      if (Tj == nullptr) {
        RankOut o = rank_out(M, r);
        o.hi = at(P.tt_hi[j]);
        o.lo = at(P.tt_lo[j]);
        o.ld = M8;
        o.hilo_f16 = f16 ? 1 : 0;
        o.scale = d->s;
        LORA_TRY(rank_T(d, P, Xl[j], Ap[j], o, ws, status, st, masks[j]));
      }
    }
    // 3. U = dZ B by a rank pass: bf16 s U (LoRA K-block of dX) and (s U)^T hi/lo (dA).
    //    Identity with r <= 32: the same pass over dZ = dY also gives dB = dZ^T (sT).
    if (P.dual) {
      RankOut uo = rank_out(M, r);
      uo.s16 = static_cast<__nv_bfloat16*>(at(P.s16[0]));
      uo.hi = at(P.ut_hi[0]);
      uo.lo = at(P.ut_lo[0]);
      uo.ld = M8;
      uo.scale = d->s;
      RankOut bo = rank_out(static_cast<int>(d->d_out), r);
      bo.f32 = dBp[0];
      LORA_TRY(run_rank2d(dZ[0], d->d_out, M, r, RP, at(P.bt[0]), at(P.tt_hi[0]), at(P.tt_lo[0]), M8, P.sp_dual,
                          static_cast<float*>(at(P.part_u)), static_cast<float*>(at(P.part_b)), uo, bo, status, st));
    }
    for (int j = 0; j < np && !P.dual; ++j) {
      RankJob J;
      J.f16 = f16;
      J.a[0] = dZ[j];
      J.a[1] = dZlo[j];
      J.na = f16 ? 2 : 1;
      J.npairs = f16 ? 2 : 1;
      J.pa[1] = 1;   // dZ_lo B
      J.a_inner = d->d_out;
      J.a_outer = M;
      J.a_ld = d->d_out;
      J.b[0] = at(P.bt[j]);
      J.b_inner = d->d_out;
      J.b_ld = d->d_out;
      J.rows = M;
      J.K = static_cast<int>(d->d_out);
      J.partial = static_cast<float*>(at(P.part_u));
      J.splits = P.splits_u;
      J.out = rank_out(M, r);
      J.out.s16 = static_cast<__nv_bfloat16*>(at(P.s16[j]));
      J.out.hi = at(P.ut_hi[j]);
      J.out.lo = at(P.ut_lo[j]);
      J.out.ld = M8;
      J.out.scale = d->s;
      LORA_TRY(run_rank_gemm(J, RP, r, status, st));
      LORA_TRY(finish_rank(&J, nullptr, RP, st));
    }
  }

  // 4. dX = [dZ | sU] [W ; A]
  const bool drop_in_gemm = masks[0] != nullptr && np == 1 && r > 0 && dXf == nullptr;
  {
    MmaParams p;
    std::memset(&p, 0, sizeof(p));
    const bool pair = pair_kernel_enabled() && M > 128;
    bool ok = true;
    for (int j = 0; j < np; ++j) {
      ok = ok && make_tm(&p.tm_a[j], dZ[j], d->d_out, M, d->d_out, 64, 128, f16);
      ok = ok && make_tm(&p.tm_w[j], Wmain[j], d->d_in, d->d_out, d->d_in, 64, 64, f16);   // MN-major
      if (r > 0) {
        ok = ok && make_tm(&p.tm_la[j], at(P.s16[j]), r, M, r, 64, 128);
        ok = ok && make_tm(&p.tm_lb[j], Ap[j], d->d_in, r, d->d_in, 64, 64);
      }
    }
    p.b_mn = 1;
    if (!ok) return LORA_ERR_CUDA;
    p.M = M;
    p.N = static_cast<int>(d->d_in);
    p.K = static_cast<int>(d->d_out);
    // Dropout with one projection: the LoRA K-blocks form s'U A in the
    // accumulator first, its dropped entries are zeroed in tensor memory, and
    // the main K-blocks accumulate on top (kMEpiGradDrop).  SwiGLU (two masks
    // on one accumulator) runs without the LoRA K-blocks and
    // dx_dropout_kernel adds the masked terms after the GEMM.
    p.lora_ksteps = (masks[0] != nullptr && !drop_in_gemm) ? 0 : (r + 15) / 16;
    if (drop_in_gemm) p.drop.mask = masks[0];
    p.out = static_cast<__nv_bfloat16*>(dX);
    p.out_f32 = dXf;
    p.out_acc = dXf_acc;
    p.z_save = nullptr;
    p.status = status;
    p.m_tiles = static_cast<int>(ceil_div(M, pair ? 256 : 128));
    p.n_tiles = static_cast<int>(ceil_div(d->d_in, 256));
    p.num_tiles = p.m_tiles * p.n_tiles;
    set_raster(p, pair, 2.0 * np * M * d->d_out, 2.0 * np * d->d_out * d->d_in);
    timing_begin(1, st);
    lora_status_t rs;
    if (drop_in_gemm) {
      rs = f16 ? launch_mma_any<true, 1, kMEpiGradF16Drop>(pair, p, dev.sms, st)
               : launch_mma_any<true, 1, kMEpiGradDrop>(pair, p, dev.sms, st);
    } else if (dXf != nullptr) {
      // fp32 dX (the attention-input block's summed input gradients): the
      // staged epilogue
      if (np != 1) return LORA_ERR_UNSUPPORTED;
      rs = f16 ? launch_mma_any<true, 1, kMEpiGradF16F32>(pair, p, dev.sms, st)
               : launch_mma_any<true, 1, kMEpiGradF32>(pair, p, dev.sms, st);
    } else if (f16) {
      if (np == 2) rs = launch_mma_any<true, 2, kMEpiGradF16>(pair, p, dev.sms, st);
      else rs = launch_mma_any<true, 1, kMEpiGradF16>(pair, p, dev.sms, st);
    } else {
      rs = launch_mma_any<true, 1, kMEpiGrad>(pair, p, dev.sms, st);
    }
    timing_end(1, st);
    LORA_TRY(rs);
  }
  if (r == 0) return LORA_OK;
  if (masks[0] != nullptr && !drop_in_gemm) {
    // dX += sum_j mask_j * (s' U_j A_j), from the (s' U_j)^T hi/lo of the U pass
    DxDropoutJob jb[2];
    for (int j = 0; j < 2; ++j) {
      const int jj = j < np ? j : 0;
      jb[j].mask = masks[jj];
      jb[j].ut_hi = static_cast<const __nv_bfloat16*>(at(P.ut_hi[jj]));
      jb[j].ut_lo = static_cast<const __nv_bfloat16*>(at(P.ut_lo[jj]));
      jb[j].A = static_cast<const __nv_bfloat16*>(Ap[jj]);
    }
    const long long tiles = ceil_div(M, kDxRows) * ceil_div(d->d_in, kDxCols);
    const int grid = static_cast<int>(tiles < static_cast<long long>(dev.sms) * 8 ? tiles : dev.sms * 8);
    const size_t smem = dx_dropout_smem_bytes(r);   // <= 65 KB at r = 128
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(dx_dropout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return cuda_error("cudaFuncSetAttribute(dx_dropout)");
    launch_k(dx_dropout_kernel, dim3(grid), dim3(256), smem, st, false, static_cast<__nv_bfloat16*>(dX), M,
             static_cast<int>(d->d_in), r, M8, jb[0], jb[1], np);
    LORA_TRY(check_launch("dx_dropout_kernel"));
  }

  // 5. dA^T = X^T (s U) (hi/lo operand) in one pass over X; without the fused
  //    pass above, dB = dZ^T (s T) too, hi/lo operands, split over tokens
  for (int j = 0; j < np; ++j) {
    RankOut ao = rank_out(static_cast<int>(d->d_in), r);
    ao.f32 = dAp[j];
    ao.transpose_f32 = 1;
    LORA_TRY(run_rank2d(Xl[j], d->d_in, M, r, RP, nullptr, at(P.ut_hi[j]), at(P.ut_lo[j]), M8, P.sp_a, nullptr,
                        static_cast<float*>(at(P.part_a)), rank_out(M, r), ao, status, st, masks[j]));
    if (P.dual) continue;
    RankJob Jb;
    Jb.a_mn = true;
    Jb.f16 = f16;
    Jb.a[0] = dZ[j];
    Jb.a[1] = dZlo[j];
    Jb.na = f16 ? 2 : 1;
    Jb.a_inner = d->d_out;
    Jb.a_outer = M;
    Jb.a_ld = d->d_out;
    Jb.b[0] = at(P.tt_hi[j]);
    Jb.b[1] = at(P.tt_lo[j]);
    Jb.nb = 2;
    Jb.b_inner = M;
    Jb.b_ld = M8;
    // dZ_hi (T_hi + T_lo) [+ dZ_lo T_hi]
    Jb.npairs = f16 ? 3 : 2;
    Jb.pb[1] = 1;
    Jb.pa[2] = 1;
    Jb.pb[2] = 0;
    Jb.rows = static_cast<int>(d->d_out);
    Jb.K = M;
    Jb.partial = static_cast<float*>(at(P.part_b));
    Jb.splits = P.splits_b;
    Jb.out = rank_out(static_cast<int>(d->d_out), r);
    Jb.out.f32 = dBp[j];
    LORA_TRY(run_rank_gemm(Jb, RP, r, status, st));
    LORA_TRY(finish_rank(&Jb, nullptr, RP, st));
  }
  return LORA_OK;
}

// ---------------------------------------------------------------------------
// Forward for callers that cannot allocate device memory: the workspace is a
// file-scope device array (every device that loads this library holds it until
// exit).  Its device address is looked up once per device, on that device's
// first call, with the device current.
// ---------------------------------------------------------------------------
}  // extern "C"

static __device__ __align__(256) unsigned char g_noalloc_scratch[LORA_LINEAR_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

lora_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_error("cudaGetDevice");
  if (dev < 0 || dev >= 64) {
    LORA_LOG("fwd_noalloc: device ordinal %d is beyond the 64 devices whose scratch address is cached", dev);
    return LORA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      LORA_LOG("cudaGetSymbolAddress(scratch) on device %d: %s", dev, cudaGetErrorString(e));
      return LORA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LORA_OK;
}
}  // namespace

extern "C" {

lora_status_t lora_linear_bwd(const lora_linear_desc* d, const void* dY, const void* X, const void* W, const void* A,
                              const void* B, const void* W_up, const void* A_up, const void* B_up,
                              const float* T_save, const float* Z_save, void* dX, float* dA, float* dB,
                              float* dA_up, float* dB_up, void* workspace, size_t workspace_bytes, void* stream) {
  const void* Xl[2] = {X, X};
  const uint8_t* masks[2] = {nullptr, nullptr};
  return bwd_core(d, dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up, workspace,
                  workspace_bytes, stream, Xl, masks);
}

lora_status_t lora_linear_fwd_noalloc(const lora_linear_desc* d, const void* X, const void* W, const void* A,
                                      const void* B, const void* W_up, const void* A_up, const void* B_up, void* Y,
                                      float* T_save, float* Z_save, void* stream) {
  // the same argument and device checks as lora_linear_fwd, in the same
  // order, before the scratch is touched
  LORA_TRY(fwd_check_args(d, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save));
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  const size_t need = make_plan(d, false).total;
  if (need > LORA_LINEAR_NOALLOC_SCRATCH_BYTES) {
    LORA_LOG("fwd_noalloc: needs %zu bytes of scratch, the static array holds %u", need,
             LORA_LINEAR_NOALLOC_SCRATCH_BYTES);
    return LORA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  LORA_TRY(noalloc_scratch(&ws));
  // The header (status word) must start at zero; everything
  // else the forward writes before it reads.
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return cuda_error("cudaMemsetAsync(scratch status)");
  return lora_linear_fwd(d, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, ws, LORA_LINEAR_NOALLOC_SCRATCH_BYTES,
                         stream);
}

lora_status_t lora_linear_noalloc_status(void* stream, uint32_t* out_status) {
  if (out_status == nullptr) return LORA_ERR_INVALID_ARG;
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  void* ws = nullptr;
  LORA_TRY(noalloc_scratch(&ws));
  return lora_linear_device_status(ws, stream, out_status);
}

// ---------------------------------------------------------------------------
// 4-bit frozen base weight ("w4g64", lora_w4.cuh)
// ---------------------------------------------------------------------------

size_t lora_linear_workspace_size_w4(const lora_linear_desc* desc, int for_backward) {
  if (check_desc(desc) != LORA_OK || desc->d_in % kW4Group != 0) return 0;
  const size_t base = align_up(lora_linear_workspace_size(desc, for_backward), 256);
  return base + w4_expand_bytes(desc, for_backward != 0);
}

lora_status_t lora_linear_dequant_w4(const void* Wq, const void* Ws, int64_t d_out, int64_t d_in, void* W,
                                     void* stream) {
  if (Wq == nullptr || Ws == nullptr || W == nullptr || d_out <= 0 || d_in <= 0) return LORA_ERR_INVALID_ARG;
  if (d_in % kW4Group != 0 || d_out % 8 != 0 || !aligned16(Wq) || !aligned16(Ws) || !aligned16(W))
    return LORA_ERR_ALIGNMENT;
  if (d_out > (int64_t(1) << 30) || d_in > (int64_t(1) << 30)) return LORA_ERR_UNSUPPORTED;
  DevInfo dev;
  LORA_TRY(device_info(&dev));
  if (dev.major != 10 || dev.minor != 0) return LORA_ERR_ARCH;
  return dequant_w4(Wq, Ws, d_out, d_in, W, static_cast<cudaStream_t>(stream));
}

lora_status_t lora_linear_fwd_w4(const lora_linear_desc* d, const void* X, const void* Wq, const void* Ws,
                                 const void* A, const void* B, const void* Wq_up, const void* Ws_up, const void* A_up,
                                 const void* B_up, void* Y, float* T_save, float* Z_save, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  LORA_TRY(check_w4(d, Wq, Ws, Wq_up, Ws_up));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  if (d->M > 0 && (X == nullptr || Y == nullptr)) return LORA_ERR_INVALID_ARG;
  if (d->r > 0 && (A == nullptr || B == nullptr)) return LORA_ERR_INVALID_ARG;
  if (swiglu && d->r > 0 && (A_up == nullptr || B_up == nullptr)) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, A, B, A_up, B_up, Y, T_save, Z_save};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  const size_t base = align_up(lora_linear_workspace_size(d, 0), 256);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, base + w4_expand_bytes(d, false), &dev));
  if (d->M == 0) return LORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (small_m_applies(d)) {
    const Plan P = make_plan(d, false);
    return run_small_m_fwd(d, P.sm_nt, X, nullptr, Wq, Ws, A, B, Y, T_save, Z_save, reinterpret_cast<uint32_t*>(ws),
                           st);
  }
  // Many tokens: expand the weight(s) to bf16 once, then the bf16 layer.
  uint8_t* Wd = ws + base;
  uint8_t* Wd_up = swiglu ? Wd + static_cast<size_t>(d->d_out) * d->d_in * 2 : nullptr;
  LORA_TRY(dequant_w4(Wq, Ws, d->d_out, d->d_in, Wd, st));
  if (swiglu) LORA_TRY(dequant_w4(Wq_up, Ws_up, d->d_out, d->d_in, Wd_up, st));
  return lora_linear_fwd(d, X, Wd, A, B, Wd_up, A_up, B_up, Y, T_save, Z_save, workspace, base, stream);
}

lora_status_t lora_linear_bwd_w4(const lora_linear_desc* d, const void* dY, const void* X, const void* Wq,
                                 const void* Ws, const void* A, const void* B, const void* Wq_up, const void* Ws_up,
                                 const void* A_up, const void* B_up, const float* T_save, const float* Z_save, void* dX,
                                 float* dA, float* dB, float* dA_up, float* dB_up, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  LORA_TRY(check_w4(d, Wq, Ws, Wq_up, Ws_up));
  const bool swiglu = d->act == LORA_ACT_SWIGLU;
  const size_t base = align_up(lora_linear_workspace_size(d, 1), 256);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, base + w4_expand_bytes(d, true), &dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Wd = ws + base;
  uint8_t* Wd_up = swiglu ? Wd + static_cast<size_t>(d->d_out) * d->d_in * 2 : nullptr;
  if (d->M > 0) {
    LORA_TRY(dequant_w4(Wq, Ws, d->d_out, d->d_in, Wd, st));
    if (swiglu) LORA_TRY(dequant_w4(Wq_up, Ws_up, d->d_out, d->d_in, Wd_up, st));
  }
  // the bf16 backward checks the remaining arguments (with M == 0 it only
  // zero-fills dA and dB and never reads the expanded weight)
  return lora_linear_bwd(d, dY, X, Wd, A, B, Wd_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up, workspace,
                         base, stream);
}

// ---------------------------------------------------------------------------
// dropout on the adapter branch's input (lora_dropout.cuh)
// ---------------------------------------------------------------------------
size_t lora_linear_workspace_size_dropout(const lora_linear_desc* desc, int for_backward) {
  if (check_desc(desc) != LORA_OK) return 0;
  return align_up(dropout_base_bytes(desc, for_backward != 0), 256);
}

lora_status_t lora_linear_fwd_dropout(const lora_linear_desc* d, const void* X, const void* W, const void* A,
                                      const void* B, const void* W_up, const void* A_up, const void* B_up,
                                      const void* mask, const void* mask_up, float p_drop, void* Y, float* T_save,
                                      float* Z_save, void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_desc(d));
  if (d->r == 0)   // no adapter: nothing to drop
    return lora_linear_fwd(d, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, workspace, workspace_bytes, stream);
  LORA_TRY(check_dropout(d, X, mask, mask_up, p_drop));
  lora_linear_desc d2 = *d;
  d2.s = d->s / (1.0f - p_drop);
  const size_t base = align_up(dropout_base_bytes(d, false), 256);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, base, &dev));
  if (d->M == 0) return LORA_OK;
  // the T pass reads X and applies the mask to its tiles in shared memory:
  // no masked copy of X in the forward
  const void* Xl[2] = {X, X};
  const uint8_t* fm[2] = {static_cast<const uint8_t*>(mask),
                          static_cast<const uint8_t*>(d->act == LORA_ACT_SWIGLU ? mask_up : mask)};
  return fwd_core(&d2, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, workspace, base, stream, Xl, false, nullptr,
                  fm);
}

lora_status_t lora_linear_bwd_dropout(const lora_linear_desc* d, const void* dY, const void* X, const void* W,
                                      const void* A, const void* B, const void* W_up, const void* A_up,
                                      const void* B_up, const void* mask, const void* mask_up, float p_drop,
                                      const float* T_save, const float* Z_save, void* dX, float* dA, float* dB,
                                      float* dA_up, float* dB_up, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  LORA_TRY(check_desc(d));
  if (d->r == 0)
    return lora_linear_bwd(d, dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up, workspace,
                           workspace_bytes, stream);
  LORA_TRY(check_dropout(d, X, mask, mask_up, p_drop));
  lora_linear_desc d2 = *d;
  d2.s = d->s / (1.0f - p_drop);
  const size_t base = align_up(dropout_base_bytes(d, true), 256);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, base, &dev));
  // the rank passes read X and apply the mask to their tiles in shared
  // memory; the dX GEMM adds the masked LoRA term in its epilogue
  const void* Xl[2] = {X, X};
  const uint8_t* masks[2] = {static_cast<const uint8_t*>(mask),
                             static_cast<const uint8_t*>(mask_up != nullptr ? mask_up : mask)};
  return bwd_core(&d2, dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up, workspace, base,
                  stream, Xl, masks);
}

// 4-bit weight, tiled code layout for the few-token forward (lora_w4.cuh)
size_t lora_linear_w4_tiled_bytes(int64_t d_out, int64_t d_in) {
  if (d_out <= 0 || d_in <= 0 || d_in % kW4Group != 0) return 0;
  return static_cast<size_t>((d_out + 127) / 128) * static_cast<size_t>(d_in / kW4Group) * kW4TileBytes;
}

lora_status_t lora_linear_w4_tile(const void* Wq, int64_t d_out, int64_t d_in, void* Wt, void* stream) {
  if (Wq == nullptr || Wt == nullptr || d_out <= 0 || d_in <= 0) return LORA_ERR_INVALID_ARG;
  if (d_in % kW4Group != 0 || !aligned16(Wq) || !aligned16(Wt)) return LORA_ERR_ALIGNMENT;
  if (d_out > (int64_t(1) << 30) || d_in > (int64_t(1) << 30)) return LORA_ERR_UNSUPPORTED;
  DevInfo dev;
  LORA_TRY(device_info(&dev));
  if (dev.major != 10 || dev.minor != 0) return LORA_ERR_ARCH;
  const long long n16 = static_cast<long long>(lora_linear_w4_tiled_bytes(d_out, d_in) / 16);
  launch_k(tile_w4_kernel, dim3(grid_for(n16, 256, dev.sms)), dim3(256), 0, static_cast<cudaStream_t>(stream), false,
           static_cast<const uint8_t*>(Wq), static_cast<long long>(d_out), static_cast<int>(d_in),
           static_cast<uint8_t*>(Wt));
  return check_launch("tile_w4_kernel");
}

lora_status_t lora_linear_fwd_w4_tiled(const lora_linear_desc* d, const void* X, const void* Wt, const void* Ws,
                                       const void* A, const void* B, void* Y, float* T_save, float* Z_save,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_w4(d, Wt, Ws, nullptr, nullptr));
  if (d->M != 0 && !small_m_applies(d)) return LORA_ERR_UNSUPPORTED;
  if (d->M > 0 && (X == nullptr || Y == nullptr)) return LORA_ERR_INVALID_ARG;
  if (A == nullptr || B == nullptr) return LORA_ERR_INVALID_ARG;
  const void* ptrs[] = {X, A, B, Y, T_save, Z_save};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return LORA_ERR_ALIGNMENT;
  const Plan P = make_plan(d, false);
  DevInfo dev;
  LORA_TRY(common_checks(d, workspace, workspace_bytes, P.total, &dev));
  if (d->M == 0) return LORA_OK;
  return run_small_m_fwd(d, P.sm_nt, X, nullptr, nullptr, Ws, A, B, Y, T_save, Z_save,
                         reinterpret_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream), Wt);
}

// RMSNorm prologue and rotary-embedding epilogue (lora_norm_rope.cuh)
lora_status_t lora_linear_rmsnorm_fwd(const void* X, const void* g, int64_t M, int64_t d, float eps, void* Xn,
                                      float* rstd, void* stream) {
  if (M < 0 || d <= 0 || !std::isfinite(eps) || eps < 0.0f || g == nullptr) return LORA_ERR_INVALID_ARG;
  if (M > 0 && (X == nullptr || Xn == nullptr || rstd == nullptr)) return LORA_ERR_INVALID_ARG;
  if (d % 8 != 0 || !aligned16(g) || (X != nullptr && !aligned16(X)) || (Xn != nullptr && !aligned16(Xn)) ||
      (reinterpret_cast<uintptr_t>(rstd) & 3u) != 0)
    return LORA_ERR_ALIGNMENT;
  if (d > (int64_t(1) << 24) || M > (int64_t(1) << 40)) return LORA_ERR_UNSUPPORTED;
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  if (M == 0) return LORA_OK;
  launch_k(rmsnorm_fwd_kernel, dim3(norm_grid(M, dev)), dim3(32 * kNormWarps), 0, static_cast<cudaStream_t>(stream),
           false, static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(g),
           static_cast<long long>(M), static_cast<int>(d), static_cast<double>(eps), static_cast<__nv_bfloat16*>(Xn),
           rstd);
  return check_launch("rmsnorm_fwd_kernel");
}

lora_status_t lora_linear_rmsnorm_bwd(const void* X, const void* g, const float* rstd, const float* dXn, int64_t M,
                                      int64_t d, void* dX, void* stream) {
  if (M < 0 || d <= 0 || g == nullptr) return LORA_ERR_INVALID_ARG;
  if (M > 0 && (X == nullptr || rstd == nullptr || dX == nullptr || dXn == nullptr)) return LORA_ERR_INVALID_ARG;
  if (d % 8 != 0 || !aligned16(g) || (X != nullptr && !aligned16(X)) || (dX != nullptr && !aligned16(dX)) ||
      (dXn != nullptr && !aligned16(dXn)) || (reinterpret_cast<uintptr_t>(rstd) & 3u) != 0)
    return LORA_ERR_ALIGNMENT;
  if (d > (int64_t(1) << 24) || M > (int64_t(1) << 40)) return LORA_ERR_UNSUPPORTED;
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  if (M == 0) return LORA_OK;
  launch_k(rmsnorm_bwd_kernel, dim3(norm_grid(M, dev)), dim3(32 * kNormWarps), 0, static_cast<cudaStream_t>(stream),
           false, static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(g), rstd, dXn,
           static_cast<long long>(M), static_cast<int>(d), static_cast<__nv_bfloat16*>(dX));
  return check_launch("rmsnorm_bwd_kernel");
}

size_t lora_linear_workspace_size_rope(const lora_linear_desc* desc, int for_backward) {
  if (check_desc(desc) != LORA_OK || desc->act != LORA_ACT_IDENTITY) return 0;
  const size_t fwd = make_plan(desc, false, false).total;
  if (!for_backward) return fwd;
  const size_t rot = make_plan(desc, true, true, true).total;    // rotated: fp16 dZ operands
  const size_t plain = make_plan(desc, true).total;              // not rotated (rope == NULL)
  const size_t bwd = rot > plain ? rot : plain;
  return bwd > fwd ? bwd : fwd;
}

lora_status_t lora_linear_fwd_rope(const lora_linear_desc* d, const lora_rope_desc* rope, const void* X,
                                   const void* W, const void* A, const void* B, void* Y, float* T_save,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_desc(d));
  RopeTables t;
  LORA_TRY(check_rope(d, rope, &t));
  const void* Xl[2] = {X, X};
  return fwd_core(d, X, W, A, B, nullptr, nullptr, nullptr, Y, T_save, nullptr, workspace, workspace_bytes, stream,
                  Xl, false, &t);
}

lora_status_t lora_linear_bwd_rope(const lora_linear_desc* d, const lora_rope_desc* rope, const void* dY,
                                   const void* X, const void* W, const void* A, const void* B, const float* T_save,
                                   float* dXn, int accumulate, float* dA, float* dB, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  LORA_TRY(check_desc(d));
  if (d->act != LORA_ACT_IDENTITY) return LORA_ERR_UNSUPPORTED;
  if (accumulate != 0 && accumulate != 1) return LORA_ERR_INVALID_ARG;
  if (d->M > 0 && dXn == nullptr) return LORA_ERR_INVALID_ARG;
  RopeTables t;
  if (rope != nullptr) LORA_TRY(check_rope(d, rope, &t));
  const void* Xl[2] = {X, X};
  const uint8_t* masks[2] = {nullptr, nullptr};
  return bwd_core(d, dY, X, W, A, B, nullptr, nullptr, nullptr, T_save, nullptr, nullptr, dA, dB, nullptr, nullptr,
                  workspace, workspace_bytes, stream, Xl, masks, rope != nullptr ? &t : nullptr, dXn, accumulate);
}


// ---------------------------------------------------------------------------
// Output projection fused with the cross-entropy loss (lora_ce.cuh and the
// kMEpiCeFwd / kMEpiCeGrad epilogues of lora_mma.cuh)
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

// Tokens per backward chunk: the chunk's bf16 logit gradient [chunk x V] is
// the only per-token buffer of the backward (2.1 GB at 8192 tokens and
// V = 128256), and the dH GEMM of a chunk of 8192 tokens at d = 4096 has 512
// CTA-pair tiles (7 waves of 74 pairs).
constexpr int64_t kCeChunkTokens = 8192;

struct CePlan {
  int n_tiles = 0;        // 256-column vocabulary tiles
  int64_t chunk = 0;      // tokens per backward (or fused) chunk
  size_t part = 0, zlab = 0, loss_tok = 0, scale = 0, dz = 0, zf = 0, total = 0;
};

lora_status_t check_ce_desc(const lora_ce_desc* d) {
  if (d == nullptr) return LORA_ERR_INVALID_ARG;
  if (d->M < 0 || d->d <= 0 || d->V <= 0) return LORA_ERR_INVALID_ARG;
  if (d->M > (int64_t(1) << 31) - 1 || d->d > (int64_t(1) << 30) || d->V > (int64_t(1) << 30))
    return LORA_ERR_UNSUPPORTED;
  if (d->d % 8 != 0 || d->V % 8 != 0) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

// mode 0: forward; 1: backward; 2: fused forward + backward (per chunk: the
// forward's partials, the chunk's fp32 logits and bf16 gradient).
CePlan ce_plan(const lora_ce_desc* d, int mode) {
  CePlan P;
  const int64_t M = d->M > 0 ? d->M : 1;
  P.n_tiles = static_cast<int>(ceil_div(d->V, 256));
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  if (mode == 2) {
    P.chunk = M < kCeChunkTokens ? M : kCeChunkTokens;
    P.part = take(static_cast<size_t>(2 * P.n_tiles) * P.chunk * sizeof(float2));
    P.zlab = take(static_cast<size_t>(P.chunk) * 4);
    P.loss_tok = take(static_cast<size_t>(M) * 4);
    P.scale = take(4);
    P.zf = take(static_cast<size_t>(P.chunk) * d->V * 4);
    P.dz = take(static_cast<size_t>(P.chunk) * d->V * 2);
  } else if (mode == 0) {
    P.part = take(static_cast<size_t>(2 * P.n_tiles) * M * sizeof(float2));
    P.zlab = take(static_cast<size_t>(M) * 4);
    P.loss_tok = take(static_cast<size_t>(M) * 4);
  } else {
    P.scale = take(4);
    P.chunk = M < kCeChunkTokens ? M : kCeChunkTokens;
    P.dz = take(static_cast<size_t>(P.chunk) * d->V * 2);
  }
  P.total = off;
  return P;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// The logits GEMM of rows [0, M) of H against all of W: forward (kMEpiCeFwd)
// or gradient recompute (kMEpiCeGrad).
template <int kEpi>
lora_status_t ce_logit_gemm(const void* H, const void* W, int64_t M, int64_t d, int64_t V, const CeParams& ce,
                            void* dz, uint32_t* status, int sms, cudaStream_t st, float* zf = nullptr) {
  MmaParams p;
  std::memset(&p, 0, sizeof(p));
  const bool pair = pair_kernel_enabled() && M > 128;
  if (!make_tm(&p.tm_a[0], H, d, M, d, 64, 128) || !make_tm(&p.tm_w[0], W, d, V, d, 64, pair ? 128 : 256))
    return LORA_ERR_CUDA;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(V);
  p.K = static_cast<int>(d);
  p.lora_ksteps = 0;
  p.out = static_cast<__nv_bfloat16*>(dz);
  p.out_f32 = zf;
  p.status = status;
  p.ce = ce;
  p.m_tiles = static_cast<int>(ceil_div(M, pair ? 256 : 128));
  p.n_tiles = static_cast<int>(ceil_div(V, 256));
  p.num_tiles = p.m_tiles * p.n_tiles;
  set_raster(p, pair, 2.0 * M * d, 2.0 * V * d);
  timing_begin(0, st);
  const lora_status_t rs = launch_mma_any<false, 1, kEpi>(pair, p, sms, st);
  timing_end(0, st);
  return rs;
}

// dH [C x d] = dz [C x V] W [V x d]: K = V, W read in place as the MN-major
// operand.
lora_status_t ce_dh_gemm(const void* dz, const void* W, int64_t C, int64_t dm, int64_t V, void* dHc, uint32_t* status,
                         int sms, cudaStream_t st) {
  MmaParams g;
  std::memset(&g, 0, sizeof(g));
  const bool pair = pair_kernel_enabled() && C > 128;
  if (!make_tm(&g.tm_a[0], dz, V, C, V, 64, 128) || !make_tm(&g.tm_w[0], W, dm, V, dm, 64, 64)) return LORA_ERR_CUDA;
  g.b_mn = 1;
  g.M = static_cast<int>(C);
  g.N = static_cast<int>(dm);
  g.K = static_cast<int>(V);
  g.lora_ksteps = 0;
  g.out = static_cast<__nv_bfloat16*>(dHc);
  g.status = status;
  g.m_tiles = static_cast<int>(ceil_div(C, pair ? 256 : 128));
  g.n_tiles = static_cast<int>(ceil_div(dm, 256));
  g.num_tiles = g.m_tiles * g.n_tiles;
  set_raster(g, pair, 2.0 * C * V, 2.0 * V * dm);
  timing_begin(1, st);
  const lora_status_t rs = launch_mma_any<true, 1, kMEpiGrad>(pair, g, sms, st);
  timing_end(1, st);
  return rs;
}

}  // namespace

extern "C" {

size_t lora_linear_ce_workspace_size(const lora_ce_desc* desc, int for_backward) {
  if (check_ce_desc(desc) != LORA_OK) return 0;
  if (for_backward == 2) return ce_plan(desc, 2).total;
  const size_t fwd = ce_plan(desc, 0).total;
  if (for_backward == 0) return fwd;
  const size_t bwd = ce_plan(desc, 1).total;
  return bwd > fwd ? bwd : fwd;
}

lora_status_t lora_linear_ce_fwd(const lora_ce_desc* d, const void* H, const void* W, const int32_t* labels,
                                 float* loss, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  LORA_TRY(check_ce_desc(d));
  if (W == nullptr || loss == nullptr || (d->M > 0 && (H == nullptr || labels == nullptr || lse == nullptr)))
    return LORA_ERR_INVALID_ARG;
  if ((H && !aligned16(H)) || !aligned16(W) || (labels && !aligned4(labels)) || !aligned4(loss) ||
      (lse && !aligned4(lse)))
    return LORA_ERR_ALIGNMENT;
  const CePlan P = ce_plan(d, 0);
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  if (workspace == nullptr || workspace_bytes < P.total || !aligned16(workspace)) return LORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->M == 0) {   // no token: the mean over no valid token is 0
    if (cudaMemsetAsync(loss, 0, sizeof(float), st) != cudaSuccess) return cuda_error("cudaMemsetAsync(loss)");
    return LORA_OK;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  CeParams ce{};
  ce.labels = labels;
  ce.part = reinterpret_cast<float2*>(ws + P.part);
  ce.zlab = reinterpret_cast<float*>(ws + P.zlab);
  // 1. logits tile by tile on the tensor cores; per token and 128-column block
  //    the epilogue keeps (max, sum exp) and the label's logit
  LORA_TRY(ce_logit_gemm<kMEpiCeFwd>(H, W, d->M, d->d, d->V, ce, nullptr, status, dev.sms, st));
  // 2. lse and each token's loss; 3. the mean over valid tokens
  const int M = static_cast<int>(d->M);
  launch_k(ce_combine_kernel, dim3(grid_for(M, kCeCombineTokens, dev.sms)), dim3(256), 0, st, false,
           static_cast<const float2*>(ce.part), 2 * P.n_tiles, M, static_cast<int>(d->V), labels,
           static_cast<const float*>(ce.zlab), lse, reinterpret_cast<float*>(ws + P.loss_tok), status);
  LORA_TRY(check_launch("ce_combine_kernel"));
  launch_k(ce_mean_kernel, dim3(1), dim3(kCeMeanThreads), 0, st, false,
           static_cast<const float*>(reinterpret_cast<float*>(ws + P.loss_tok)), labels, M, static_cast<int>(d->V),
           loss);
  return check_launch("ce_mean_kernel");
}

lora_status_t lora_linear_ce_bwd(const lora_ce_desc* d, const void* H, const void* W, const int32_t* labels,
                                 const float* lse, const float* dloss, void* dH, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  LORA_TRY(check_ce_desc(d));
  if (W == nullptr || dloss == nullptr ||
      (d->M > 0 && (H == nullptr || labels == nullptr || lse == nullptr || dH == nullptr)))
    return LORA_ERR_INVALID_ARG;
  if ((H && !aligned16(H)) || !aligned16(W) || (dH && !aligned16(dH)) || (labels && !aligned4(labels)) ||
      (lse && !aligned4(lse)) || !aligned4(dloss))
    return LORA_ERR_ALIGNMENT;
  const CePlan P = ce_plan(d, 1);
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  if (workspace == nullptr || workspace_bytes < P.total || !aligned16(workspace)) return LORA_ERR_WORKSPACE;
  if (d->M == 0) return LORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* scale = reinterpret_cast<float*>(ws + P.scale);
  void* dz = ws + P.dz;
  const int64_t M = d->M, dm = d->d, V = d->V;
  // 1. scale = d(loss) / (number of valid tokens)
  launch_k(ce_scale_kernel, dim3(1), dim3(kCeMeanThreads), 0, st, false, labels, static_cast<int>(M),
           static_cast<int>(V), dloss, scale, status);
  LORA_TRY(check_launch("ce_scale_kernel"));
  for (int64_t m0 = 0; m0 < M; m0 += P.chunk) {
    const int64_t C = (M - m0) < P.chunk ? (M - m0) : P.chunk;
    const void* Hc = static_cast<const uint8_t*>(H) + static_cast<size_t>(m0) * dm * 2;
    // 2. the chunk's logits again, turned into the gradient of the loss with
    //    respect to them, bf16 [C x V]
    CeParams ce{};
    ce.labels = labels + m0;
    ce.lse = lse + m0;
    ce.scale = scale;
    LORA_TRY(ce_logit_gemm<kMEpiCeGrad>(Hc, W, C, dm, V, ce, dz, status, dev.sms, st));
    // 3. dH = dz W
    LORA_TRY(ce_dh_gemm(dz, W, C, dm, V, static_cast<uint8_t*>(dH) + static_cast<size_t>(m0) * dm * 2, status,
                        dev.sms, st));
  }
  return LORA_OK;
}

lora_status_t lora_linear_ce_fwd_bwd(const lora_ce_desc* d, const void* H, const void* W, const int32_t* labels,
                                     const float* dloss, float* loss, float* lse, void* dH, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  LORA_TRY(check_ce_desc(d));
  if (W == nullptr || dloss == nullptr || loss == nullptr ||
      (d->M > 0 && (H == nullptr || labels == nullptr || lse == nullptr || dH == nullptr)))
    return LORA_ERR_INVALID_ARG;
  if ((H && !aligned16(H)) || !aligned16(W) || (dH && !aligned16(dH)) || (labels && !aligned4(labels)) ||
      (lse && !aligned4(lse)) || !aligned4(dloss) || !aligned4(loss))
    return LORA_ERR_ALIGNMENT;
  const CePlan P = ce_plan(d, 2);
  DevInfo dev;
  LORA_TRY(check_arch(&dev));
  if (workspace == nullptr || workspace_bytes < P.total || !aligned16(workspace)) return LORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->M == 0) {   // no token: the mean over no valid token is 0, and there is no dH
    if (cudaMemsetAsync(loss, 0, sizeof(float), st) != cudaSuccess) return cuda_error("cudaMemsetAsync(loss)");
    return LORA_OK;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* scale = reinterpret_cast<float*>(ws + P.scale);
  float* loss_tok = reinterpret_cast<float*>(ws + P.loss_tok);
  float* zf = reinterpret_cast<float*>(ws + P.zf);
  void* dz = ws + P.dz;
  const int64_t M = d->M, dm = d->d, V = d->V;
  // 1. scale = d(loss) / (number of valid tokens), from the labels alone
  launch_k(ce_scale_kernel, dim3(1), dim3(kCeMeanThreads), 0, st, false, labels, static_cast<int>(M),
           static_cast<int>(V), dloss, scale, status);
  LORA_TRY(check_launch("ce_scale_kernel"));
  for (int64_t m0 = 0; m0 < M; m0 += P.chunk) {
    const int C = static_cast<int>((M - m0) < P.chunk ? (M - m0) : P.chunk);
    const void* Hc = static_cast<const uint8_t*>(H) + static_cast<size_t>(m0) * dm * 2;
    // 2. the chunk's logits on the tensor cores: (max, sum exp) per
    //    128-column block and the label's logit, and the fp32 logits themselves
    CeParams ce{};
    ce.labels = labels + m0;
    ce.part = reinterpret_cast<float2*>(ws + P.part);
    ce.zlab = reinterpret_cast<float*>(ws + P.zlab);
    LORA_TRY(ce_logit_gemm<kMEpiCeFwdZ>(Hc, W, C, dm, V, ce, nullptr, status, dev.sms, st, zf));
    // 3. lse and each token's loss
    launch_k(ce_combine_kernel, dim3(grid_for(C, kCeCombineTokens, dev.sms)), dim3(256), 0, st, false,
             static_cast<const float2*>(ce.part), 2 * P.n_tiles, C, static_cast<int>(V), labels + m0,
             static_cast<const float*>(ce.zlab), lse + m0, loss_tok + m0, status);
    LORA_TRY(check_launch("ce_combine_kernel"));
    // 4. the gradient with respect to the logits, bf16 [C x V]
    const long long n8 = static_cast<long long>(C) * (V / 8);
    launch_k(ce_dz_kernel, dim3(grid_for(n8, 256, dev.sms)), dim3(256), 0, st, false,
             static_cast<const float*>(zf), C, static_cast<int>(V), labels + m0, static_cast<const float*>(lse + m0),
             static_cast<const float*>(scale), static_cast<__nv_bfloat16*>(dz));
    LORA_TRY(check_launch("ce_dz_kernel"));
    // 5. dH = dz W
    LORA_TRY(ce_dh_gemm(dz, W, C, dm, V, static_cast<uint8_t*>(dH) + static_cast<size_t>(m0) * dm * 2, status,
                        dev.sms, st));
  }
  // 6. the mean over valid tokens
  launch_k(ce_mean_kernel, dim3(1), dim3(kCeMeanThreads), 0, st, false, static_cast<const float*>(loss_tok), labels,
           static_cast<int>(M), static_cast<int>(V), loss);
  return check_launch("ce_mean_kernel");
}

}  // extern "C"
