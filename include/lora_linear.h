/*
 * lora_linear.h — C ABI of the B200 (sm_100a) fused LoRA-adapted linear layer.
 *
 * The operation (forward):
 *     T = X A^T                       rank-r intermediate, M x r
 *     Z = X W^T + s T B^T             M x d_out
 *     Y = act(Z)
 * follows "Liger-Kernel内核级优化：GPU利用率飙升至90%以上", section
 * "为什么传统微调会“卡脖子”？" (y = Wx + B(Ax) and its four-call PyTorch form
 * ax = linear(x, A); bax = linear(ax, B); wx = linear(x, W); y = wx + bax),
 * with the LoRA branch scaled by s = alpha / r, and section
 * "内核融合：把“碎片化”变成“流水线”" (activation fused after the add: SiLU).
 * SwiGLU pairs a gate and an up projection, each a LoRA linear with its own
 * W, A, B: Y = SiLU(Z_gate) * Z_up ("Swift-All一文详解：如何用Liger-Kernel提升
 * 训练效率", 2.2 (2) "SwiGLU 激活函数融合").
 *
 * The backward is the chain rule of that forward (the pages say only that it
 * is fused, with recompute: "系统架构与工作流程"):
 *     dZ = dY * act'(Z)               (identity: dZ = dY)
 *     U  = dZ B                       M x r
 *     dX = dZ W + s U A               M x d_in
 *     dA = s U^T X                    r x d_in
 *     dB = s dZ^T T                   d_out x r
 * W is frozen: there is no dW.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers marked "device" must point to memory of the current CUDA device;
 *   all of them are caller-owned.  The library allocates nothing and keeps no
 *   state between calls other than a per-device cache of the SM count (and,
 *   for lora_linear_fwd_noalloc, of its static scratch array's address).  The
 *   one exception is a debugging aid: with the environment variable
 *   LORA_LINEAR_DEBUG=2 the few-token forward allocates an 8 MB device trace
 *   buffer once (cudaMalloc) and prints per-CTA phase timestamps after each
 *   launch.  Production callers leave LORA_LINEAR_DEBUG unset (or 0/1).
 * - Matrices are dense, row-major, with no padding between rows.
 *   bf16 tensors are IEEE bfloat16 bit patterns (2 bytes per element).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and never synchronises, except
 *   lora_linear_device_status which reads the status word back.
 * - Alignment: every tensor pointer is 16-byte aligned; d_in % 8 == 0,
 *   d_out % 8 == 0; r % 8 == 0 with 0 <= r <= 128.  Violations return
 *   LORA_ERR_ALIGNMENT (pointers, strides) or LORA_ERR_UNSUPPORTED (r) before
 *   anything is launched.
 * - r == 0 is a plain linear layer: A, B (and the _up twins) may be NULL and
 *   T_save is ignored.
 * - M may be 0: the per-token tensors (X, Y, T_save, Z_save, dY, dX) are
 *   empty and may be NULL; the forward launches nothing and the backward
 *   zero-fills dA and dB.
 * - Outputs are overwritten, never accumulated into.
 * - Results: Y and dX are bf16 (round to nearest even of fp32 accumulators);
 *   T_save, Z_save, dA, dB are fp32.
 * - The device must be sm_100 (B200).  Anything else returns LORA_ERR_ARCH.
 *   There is no CPU or fallback path.
 * - The workspace holds a 32-bit device status word at offset 0.  Kernels OR
 *   error bits into it (a bounded wait that gave up, a failed device-side
 *   check); they never clear it.  Zero it once with lora_linear_workspace_init
 *   before the first call; read it with lora_linear_device_status.  Words 8
 *   to 27 of the same 256-byte header are flags of the forward GEMM (one
 *   launch sets them and zeroes them again before it ends);
 *   lora_linear_workspace_init zeroes them too.
 * - Calls that share a workspace must not overlap in time (issue them on one
 *   stream): they use the same scratch regions.
 */
#ifndef LORA_LINEAR_H
#define LORA_LINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Activation applied after the add (see the header comment). */
typedef enum lora_act_t {
    LORA_ACT_IDENTITY = 0,
    LORA_ACT_SILU = 1,
    LORA_ACT_SWIGLU = 2
} lora_act_t;

typedef enum lora_status_t {
    LORA_OK = 0,
    LORA_ERR_INVALID_ARG = 1,   /* NULL required pointer, negative size, bad act */
    LORA_ERR_ALIGNMENT = 2,     /* pointer not 16-byte aligned, d_in/d_out not multiples of 8 */
    LORA_ERR_UNSUPPORTED = 3,   /* r not a multiple of 8 or above 128; a size or option an entry point
                                   does not serve (stated with that entry point) */
    LORA_ERR_ARCH = 4,          /* current device is not sm_100 */
    LORA_ERR_WORKSPACE = 5,     /* workspace NULL or smaller than lora_linear_workspace_size */
    LORA_ERR_CUDA = 6,          /* a CUDA runtime/driver call or a launch failed */
    LORA_ERR_DEVICE_STATUS = 7  /* the device status word is non-zero */
} lora_status_t;

/* Problem description.  M tokens; X is M x d_in; W is d_out x d_in;
 * A is r x d_in; B is d_out x r; s = alpha / r; act is a lora_act_t. */
typedef struct lora_linear_desc {
    int64_t M;
    int64_t d_in;
    int64_t d_out;
    int64_t r;
    float s;
    int32_t act;
} lora_linear_desc;

/* Bytes of device workspace lora_linear_fwd (for_backward == 0) or
 * lora_linear_bwd (for_backward != 0) needs for `desc`.  Returns 0 for an
 * invalid desc.  The size is a function of the desc only, and the backward
 * size is never below the forward size, so one workspace sized for the
 * backward serves both calls (one after the other, on one stream). */
size_t lora_linear_workspace_size(const lora_linear_desc* desc, int for_backward);

/* Zero the header of a workspace (asynchronous, on `stream`): the status
 * block, whose word 0 is the status word.  Call this once after allocating
 * the workspace, and again after any call that left a non-zero status.
 * workspace_bytes must be at least the header (256 bytes). */
lora_status_t lora_linear_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, copy the workspace status word to *out_status and
 * return LORA_OK if it is zero, LORA_ERR_DEVICE_STATUS otherwise.  Bits:
 *   0x1  a bounded wait on an mbarrier gave up (the kernel stopped its work)
 *   0x2  a device-side argument check failed (e.g. a rotary position outside
 *        its table)
 *   0x4  a value converted to fp16 was outside fp16's finite range (backward
 *        with an activation, or of a rotated projection)
 * Intended for tests and debugging. */
lora_status_t lora_linear_device_status(const void* workspace, void* stream, uint32_t* out_status);

/* Forward.  Device pointers:
 *   X [M x d_in] bf16, W [d_out x d_in] bf16, A [r x d_in] bf16, B [d_out x r] bf16.
 *   W_up, A_up, B_up: the up projection's weights for LORA_ACT_SWIGLU, else NULL.
 *   Y [M x d_out] bf16 (output).
 *   T_save: NULL, or fp32 output [M x r] (SwiGLU: gate's [M x r] then up's [M x r])
 *           holding T = X A^T for the backward.
 *   Z_save: NULL, or fp32 output [M x d_out] (SwiGLU: Z_gate then Z_up, each
 *           [M x d_out]) holding the pre-activation; ignored for identity.
 *   workspace: device, >= lora_linear_workspace_size(desc, 0) bytes.
 * Launches: kernels are stream-ordered and may start while the preceding
 * kernel in the stream drains (programmatic dependent launch; each waits for
 * its predecessor before touching memory).  With 1..64 tokens, identity or
 * SiLU and r > 0 the forward is one launch of thread-block clusters (one
 * cluster of 1..16 CTAs per 128 output features; the cluster size is the
 * largest the device reports it can keep resident for every slice at once).
 * With more tokens, identity and 0 < r <= 64, it is one GEMM launch that
 * also computes T, as long as M <= 256 x (SMs / 2) (18944 on a B200): each
 * 256-row block's first output tile accumulates T = X A^T beside its main
 * product and publishes bf16(s T) in the workspace; the block's other tiles
 * wait for it (bounded, as every wait here) before their adapter K-block.
 * Otherwise a T pass (with its split-K reduction) runs before the GEMM. */
lora_status_t lora_linear_fwd(const lora_linear_desc* desc,
                              const void* X, const void* W, const void* A, const void* B,
                              const void* W_up, const void* A_up, const void* B_up,
                              void* Y, float* T_save, float* Z_save,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Backward.  Device pointers:
 *   dY [M x d_out] bf16; X, W, A, B (and the _up twins for SwiGLU) as in the forward.
 *   T_save: the forward's T_save, or NULL to recompute T = X A^T.
 *   Z_save: the forward's Z_save (required when act != identity), else NULL.
 *   dX [M x d_in] bf16 (output).
 *   dA [r x d_in] fp32, dB [d_out x r] fp32 (outputs; NULL when r == 0).
 *   dA_up, dB_up: the up projection's adapter gradients for SwiGLU, else NULL.
 *   workspace: device, >= lora_linear_workspace_size(desc, 1) bytes. */
lora_status_t lora_linear_bwd(const lora_linear_desc* desc,
                              const void* dY, const void* X, const void* W,
                              const void* A, const void* B,
                              const void* W_up, const void* A_up, const void* B_up,
                              const float* T_save, const float* Z_save,
                              void* dX, float* dA, float* dB, float* dA_up, float* dB_up,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Failure-detection self-test.  The pages have no counterpart: it checks this
 * library's own give-up path.  Launches one CTA on `stream` whose thread waits
 * on an mbarrier that nothing arrives on, through the same bounded-wait
 * routine every kernel here uses, with a limit of 2^limit_log2 SM cycles
 * instead of the usual 2^34.  The wait gives up, ORs 0x1 into the workspace
 * status word and the kernel returns: no trap, the context stays usable.
 * Read the outcome with lora_linear_device_status; clear it with
 * lora_linear_workspace_init.
 *   workspace: device, >= 256 bytes (the header), 16-byte aligned, else
 *              LORA_ERR_WORKSPACE.
 *   limit_log2: 10..30, else LORA_ERR_INVALID_ARG. */
lora_status_t lora_linear_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_log2,
                                                void* stream);

/* Static string for a status code (never NULL). */
const char* lora_status_string(lora_status_t status);

/* Library ABI version (incremented on any signature change). */
int lora_linear_abi_version(void);

/* Number of CUDA kernels this library has launched in the calling process
 * (all devices, all threads).  For accounting in benchmarks and tests. */
uint64_t lora_linear_launch_count(void);

/* Benchmark instrumentation.  lora_linear_timing_enable(1) makes every later
 * lora_linear_fwd / lora_linear_bwd call record a CUDA event pair around its
 * main GEMM launch (the tcgen05 kernel that computes Y or dX) on the call's
 * stream.  lora_linear_timing_read waits for those events, returns the summed
 * milliseconds and launch counts of the forward and backward GEMMs recorded
 * since the previous read, and resets them.  enable(0) stops recording.  The
 * event objects are created by enable(1) (up to 1024 pairs per direction);
 * further launches beyond that are not timed.  Not meant for concurrent calls
 * from several host threads. */
lora_status_t lora_linear_timing_enable(int enable);
lora_status_t lora_linear_timing_read(double* fwd_ms, uint64_t* fwd_launches, double* bwd_ms,
                                      uint64_t* bwd_launches);

/* Forward without a workspace argument, for callers that cannot allocate
 * device memory: for example a plug-in inside a host application that owns
 * every device allocation through its own pool and forbids direct cudaMalloc,
 * or a latency-critical caller that must not pay for cudaMalloc's implicit
 * synchronisation.  The pages describe no such variant; it has no counterpart
 * there.
 *
 * Same arguments, results and errors as lora_linear_fwd, minus the workspace:
 * the scratch memory lives in a file-scope device array of
 * LORA_LINEAR_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU loading this
 * library holds until the process exits.  Nothing is allocated by this call.
 * - A problem whose forward workspace (lora_linear_workspace_size(desc, 0))
 *   exceeds that size is rejected with LORA_ERR_UNSUPPORTED before anything
 *   runs.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - Every call, on every stream, shares the one array and leaves its contents
 *   behind; each call clears the part that must start at zero (its status
 *   word) and writes every other byte it reads before reading it.  Calls that
 *   overlap on the GPU (e.g. on two streams at once) race on it: serialise
 *   them.
 * - Arguments are checked in lora_linear_fwd's order (desc, pointers,
 *   alignment, device architecture, then the scratch size) before the array
 *   is touched, so a rejected call queues nothing.
 * - The cached address belongs to the device's primary context: do not use
 *   this entry point across a cudaDeviceReset of that device.  Devices with
 *   an ordinal of 64 or more are not served (LORA_ERR_UNSUPPORTED).
 * - A kernel that gives up (a bounded wait that ran out) records it in the
 *   array's status word, not in a return value: read it with
 *   lora_linear_noalloc_status after the call and before the next one (the
 *   next call clears it). */
#define LORA_LINEAR_NOALLOC_SCRATCH_BYTES (16u << 20)
lora_status_t lora_linear_fwd_noalloc(const lora_linear_desc* desc,
                                      const void* X, const void* W, const void* A, const void* B,
                                      const void* W_up, const void* A_up, const void* B_up,
                                      void* Y, float* T_save, float* Z_save, void* stream);

/* The device status word of lora_linear_fwd_noalloc's scratch array on the
 * current device (same bits as lora_linear_device_status).  Synchronises
 * `stream`, copies the word to *out_status (host) and returns LORA_OK if it is
 * zero, LORA_ERR_DEVICE_STATUS otherwise.  Call it on the stream of the
 * no-alloc call whose outcome you want, after that call and before the next
 * one.  Allocates nothing.  out_status NULL: LORA_ERR_INVALID_ARG; not sm_100:
 * LORA_ERR_ARCH.  The pages have no counterpart: it reports this library's
 * own failure detection. */
lora_status_t lora_linear_noalloc_status(void* stream, uint32_t* out_status);

/* ------------------------------------------------------------------------
 * 4-bit frozen base weight ("w4g64").  The pages name QLoRA fine-tuning, whose
 * frozen weight is stored at 4 bits, among the settings the fused kernels
 * serve ("Liger-Kernel内核级优化：GPU利用率飙升至90%以上", opening section;
 * "Swift-All一文详解：如何用Liger-Kernel提升训练效率", section 2.3, table), but
 * they give no storage format.  This library's format:
 *   Wq [d_out x d_in/2] uint8: the codes q[n][k] in 0..15, two per byte, byte
 *      j of row n holding q[n][2j] in its low nibble and q[n][2j+1] in its
 *      high nibble;
 *   Ws [d_in/64 x d_out] bf16 (group-major): Ws[g][n] scales
 *      W[n][64g .. 64g+63];
 *   W[n][k] = bf16(Ws[k/64][n] * (q[n][k] - 8)), rounded to nearest even (the
 *      product is exact in fp32).
 * The layer is the bf16 layer above on that W.  d_in must be a multiple of 64
 * (LORA_ERR_ALIGNMENT otherwise); Wq, Ws (and Wq_up, Ws_up for SwiGLU) are
 * required, device-resident, 16-byte aligned and only read.
 * ------------------------------------------------------------------------ */

/* Workspace bytes for lora_linear_fwd_w4 (for_backward = 0) or
 * lora_linear_bwd_w4 (1): the bf16 workspace plus, except for the few-token
 * forward, room to expand the weight(s) to bf16 (d_out * d_in * 2 bytes per
 * projection).  0 for an invalid desc or d_in % 64 != 0. */
size_t lora_linear_workspace_size_w4(const lora_linear_desc* desc, int for_backward);

/* Expand a 4-bit weight to bf16: W [d_out x d_in] bf16 (device, written).
 * Asynchronous on `stream`.  d_in % 64 == 0 and d_out % 8 == 0, pointers
 * 16-byte aligned (LORA_ERR_ALIGNMENT), d_out, d_in > 0 (LORA_ERR_INVALID_ARG). */
lora_status_t lora_linear_dequant_w4(const void* Wq, const void* Ws, int64_t d_out, int64_t d_in, void* W,
                                     void* stream);

/* Forward with 4-bit base weight(s).  Arguments as lora_linear_fwd, with
 * (Wq, Ws) in place of W and (Wq_up, Ws_up) in place of W_up.  With 1..64
 * tokens, identity or SiLU and 0 < r <= 64 the codes are streamed once and
 * expanded inside the few-token kernel (one launch); otherwise the weight(s)
 * are expanded into the workspace and the bf16 path runs on them.
 * workspace: >= lora_linear_workspace_size_w4(desc, 0) bytes. */
lora_status_t lora_linear_fwd_w4(const lora_linear_desc* desc, const void* X, const void* Wq, const void* Ws,
                                 const void* A, const void* B, const void* Wq_up, const void* Ws_up,
                                 const void* A_up, const void* B_up, void* Y, float* T_save, float* Z_save,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Backward with 4-bit base weight(s) (frozen: no gradient for them).
 * Arguments as lora_linear_bwd with (Wq, Ws), (Wq_up, Ws_up) in place of W,
 * W_up; the weight(s) are expanded into the workspace, then the bf16 backward
 * runs.  workspace: >= lora_linear_workspace_size_w4(desc, 1) bytes. */
lora_status_t lora_linear_bwd_w4(const lora_linear_desc* desc, const void* dY, const void* X, const void* Wq,
                                 const void* Ws, const void* A, const void* B, const void* Wq_up, const void* Ws_up,
                                 const void* A_up, const void* B_up, const float* T_save, const float* Z_save,
                                 void* dX, float* dA, float* dB, float* dA_up, float* dB_up, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Tiled code layout for the few-token forward: the codes of each 128-row x
 * 64-feature tile are 4096 contiguous bytes (row i of the tile at byte 32 i,
 * same nibble order), tiles ordered by 128-row slice, then by 64-feature
 * block: tile (g, kb) at byte (g * d_in/64 + kb) * 4096; rows past d_out are
 * zero.  A stage then loads one contiguous 4 KB block instead of 128
 * 32-byte row pieces.  The base weight is frozen, so this is a load-time
 * step.
 * lora_linear_w4_tiled_bytes: size of the tiled codes (0 if d_in % 64 != 0
 *   or a size is not positive).
 * lora_linear_w4_tile: writes Wt (device, that size) from the row-major Wq;
 *   asynchronous on `stream`; 16-byte aligned pointers.
 * lora_linear_fwd_w4_tiled: the few-token forward (1..64 tokens, identity or
 *   SiLU, 0 < r <= 64; else LORA_ERR_UNSUPPORTED; M == 0 is a no-op) on the
 *   tiled codes Wt and the scales Ws; other arguments as lora_linear_fwd;
 *   workspace >= lora_linear_workspace_size(desc, 0). */
size_t lora_linear_w4_tiled_bytes(int64_t d_out, int64_t d_in);
lora_status_t lora_linear_w4_tile(const void* Wq, int64_t d_out, int64_t d_in, void* Wt, void* stream);
lora_status_t lora_linear_fwd_w4_tiled(const lora_linear_desc* desc, const void* X, const void* Wt, const void* Ws,
                                       const void* A, const void* B, void* Y, float* T_save, float* Z_save,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dropout on the adapter branch's input.  The pages' LoRA configurations set
 * a LoRA dropout (lora_dropout = 0.05 in "Swift-All一文详解：如何用Liger-Kernel
 * 提升训练效率", section 3's training configuration; 0.1 in the usage example
 * of "企业官网建设流程全解析") without saying where it applies; the reading
 * taken is the usual one: only the adapter sees the dropped input,
 *   X_d = X * mask / (1 - p_drop),   T = X_d A^T,   Z = X W^T + s T B^T,
 * and the backward is its chain rule (dX = dZ W + mask * (s U A) / (1 - p),
 * dA = s U^T X_d, dB = s dZ^T T).  The random draws are an input:
 *   mask, mask_up: device, [M x d_in/8] bytes; bit j of byte b (least
 *     significant first) keeps element 8b + j of that token's row of X.
 *     mask_up (SwiGLU's up projection; its own draw) is required for SwiGLU,
 *     NULL otherwise.  Both may be NULL when M == 0.  Only read.
 *   p_drop: the drop probability, 0 <= p_drop < 1 (else LORA_ERR_INVALID_ARG).
 * T_save holds (X * mask) A^T, without the 1/(1 - p_drop) factor; pass it
 * back to lora_linear_bwd_dropout unchanged.  With r == 0 these calls are the
 * plain ones.  The few-token kernel is not used (dropout is a training-time
 * transform).  No masked copy of X is made: the rank passes that read X for
 * the adapter (T, dA) zero the dropped elements of each X tile in shared
 * memory.  The masked LoRA term of dX is formed on the tensor cores inside
 * the dX GEMM (one projection: the term first, its dropped entries zeroed,
 * dZ W accumulated on top) or added after it (SwiGLU).
 * ------------------------------------------------------------------------ */

/* Workspace bytes for lora_linear_fwd_dropout (0) / lora_linear_bwd_dropout
 * (1): the layer's workspace for the tiled path (the few-token forward, which
 * needs none, is not used here).  0 for an invalid desc. */
size_t lora_linear_workspace_size_dropout(const lora_linear_desc* desc, int for_backward);

lora_status_t lora_linear_fwd_dropout(const lora_linear_desc* desc, const void* X, const void* W, const void* A,
                                      const void* B, const void* W_up, const void* A_up, const void* B_up,
                                      const void* mask, const void* mask_up, float p_drop, void* Y, float* T_save,
                                      float* Z_save, void* workspace, size_t workspace_bytes, void* stream);

lora_status_t lora_linear_bwd_dropout(const lora_linear_desc* desc, const void* dY, const void* X, const void* W,
                                      const void* A, const void* B, const void* W_up, const void* A_up,
                                      const void* B_up, const void* mask, const void* mask_up, float p_drop,
                                      const float* T_save, const float* Z_save, void* dX, float* dA, float* dB,
                                      float* dA_up, float* dB_up, void* workspace, size_t workspace_bytes,
                                      void* stream);

/* ------------------------------------------------------------------------
 * RMSNorm prologue and rotary-embedding epilogue of the attention-input
 * (q, k, v) projections.  "Swift-All一文详解：如何用Liger-Kernel提升训练效率",
 * 2.2 (1) "RMSNorm + Rotary Embedding + Attention QKV 融合", gives the
 * sequence they fuse: normalise x, project it to q, k and v, rotate q and k.
 * The sketch of that kernel in "企业官网建设流程全解析" (the page's extracted
 * title), section "融合内核是如何工作的", fixes the norm (reciprocal square
 * root of the mean square plus 1e-6, times the norm's weight) and takes the
 * rotation's cosine and sine tables as arguments, indexed by the feature's
 * offset within half a head.  Readings taken:
 *   x_n = bf16(x * rstd * g),   rstd = 1 / sqrt(mean_j x_j^2 + eps)  per token,
 *     rounded once (to nearest even) from the exact value; g is frozen;
 *   q = rot(Z_q), k = rot(Z_k) with Z the identity LoRA linear of x_n; rot
 *     turns feature i of each head of head_dim features with feature
 *     i + head_dim/2 by the table angle at the token's position:
 *       (a, b) -> (a cos - b sin, b cos + a sin);
 *   the backward is the chain rule (the projections' input gradients add up
 *     before the norm's backward).
 * A block step is: lora_linear_rmsnorm_fwd; lora_linear_fwd_rope for q and k
 * and lora_linear_fwd for v, all on x_n; then lora_linear_bwd_rope for q, k
 * and v (rope NULL for v), the first writing and the others adding their
 * input gradients into one fp32 dx_n; then lora_linear_rmsnorm_bwd on dx_n.
 * dx_n is fp32 because three bf16 roundings before the sum would exceed the
 * tolerance on the near-zero entries of dx.
 * ------------------------------------------------------------------------ */

/* Rotary tables.  pos: device int32 [M], each token's position (0 <= pos <
 * n_pos; a position outside sets status bit 0x2 and leaves that token
 * unrotated), 4-byte aligned.  cos, sin: device fp32 [n_pos x head_dim/2],
 * 16-byte aligned; row p holds the angle's cosine / sine for pair i of a head
 * at position p.  head_dim: 64 or 128 (LORA_ERR_UNSUPPORTED otherwise), and a
 * divisor of d_out (LORA_ERR_INVALID_ARG).  All caller-owned, only read.
 * pos, cos, sin may be NULL when M == 0. */
typedef struct lora_rope_desc {
    const int32_t* pos;
    const float* cos;
    const float* sin;
    int64_t n_pos;
    int32_t head_dim;
} lora_rope_desc;

/* x_n = bf16(x * rstd * g) and rstd = 1 / sqrt(mean(x^2) + eps), per token.
 * X [M x d] bf16, g [d] bf16 (device, read); Xn [M x d] bf16 and rstd [M] fp32
 * (device, written; rstd is the backward's input).  The sum of squares, rstd
 * and the product are taken in fp64, and x_n is their correctly rounded bf16
 * value.  d % 8 == 0 and X, g, Xn 16-byte aligned, rstd 4-byte aligned
 * (LORA_ERR_ALIGNMENT); eps >= 0 and finite, M >= 0, d > 0
 * (LORA_ERR_INVALID_ARG).  M == 0 launches nothing.  Asynchronous on `stream`. */
lora_status_t lora_linear_rmsnorm_fwd(const void* X, const void* g, int64_t M, int64_t d, float eps, void* Xn,
                                      float* rstd, void* stream);

/* dX [M x d] bf16 = rstd (g dx_n - x_hat mean(g dx_n x_hat)), x_hat = x rstd.
 * dXn: device fp32 [M x d], the summed input gradients of the projections
 * that read x_n (lora_linear_bwd_rope's output), 16-byte aligned.  rstd: the
 * forward's output.  Alignment and errors as lora_linear_rmsnorm_fwd.  g gets
 * no gradient (frozen). */
lora_status_t lora_linear_rmsnorm_bwd(const void* X, const void* g, const float* rstd, const float* dXn, int64_t M,
                                      int64_t d, void* dX, void* stream);

/* Workspace bytes for lora_linear_fwd_rope (0) / lora_linear_bwd_rope (1); 0
 * for an invalid desc or an activation other than identity. */
size_t lora_linear_workspace_size_rope(const lora_linear_desc* desc, int for_backward);

/* Forward of a rotated projection: Y = rot(X W^T + s (X A^T) B^T), bf16, the
 * rotation applied to the fp32 accumulator in the GEMM's epilogue (one
 * rounding).  desc->act must be LORA_ACT_IDENTITY (LORA_ERR_UNSUPPORTED).
 * X is x_n.  Other arguments as lora_linear_fwd (no SwiGLU twins, no Z_save);
 * T_save holds T = X A^T for the backward.  The few-token kernel is not used.
 * As with lora_linear_fwd, r <= 64 and M <= 256 x (SMs / 2) make it one GEMM
 * launch that also computes T; otherwise a T pass runs first.
 * workspace >= lora_linear_workspace_size_rope(desc, 0). */
lora_status_t lora_linear_fwd_rope(const lora_linear_desc* desc, const lora_rope_desc* rope, const void* X,
                                   const void* W, const void* A, const void* B, void* Y, float* T_save,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Backward of a projection of the block.  rope != NULL (q, k): dZ =
 * rot^T(dY), emitted as fp16 hi + lo (a value outside fp16's range sets status
 * bit 0x4); rope == NULL (v): dZ = dY.  Then the layer's backward on dZ:
 * dx = dZ W + s U A, dA = s U^T X, dB = s dZ^T T, U = dZ B.
 * dXn: device fp32 [M x d_in], 16-byte aligned: accumulate == 0 writes dx
 * into it, accumulate == 1 adds dx to it (other values: LORA_ERR_INVALID_ARG).
 * Other arguments as lora_linear_bwd without the SwiGLU twins and Z_save;
 * desc->act must be LORA_ACT_IDENTITY (LORA_ERR_UNSUPPORTED).
 * workspace >= lora_linear_workspace_size_rope(desc, 1). */
lora_status_t lora_linear_bwd_rope(const lora_linear_desc* desc, const lora_rope_desc* rope, const void* dY,
                                   const void* X, const void* W, const void* A, const void* B, const float* T_save,
                                   float* dXn, int accumulate, float* dA, float* dB, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Output projection fused with the cross-entropy loss.  "Swift-All一文详解：
 * 如何用Liger-Kernel提升训练效率", 2.2 (3) "CrossEntropy Loss 与最后一层 Logits
 * 计算融合": the loss is computed together with the last layer's logits, in a
 * numerically stable way, and its gradient is taken straight from the
 * previous layer's output without the full probability distribution.  The
 * quantity is the usual language-model loss:
 *     z_m  = h_m W^T                         logits of token m (V classes)
 *     loss = (1/N) sum over valid m of (logsumexp(z_m) - z_m[y_m])
 *     dh_m = d(loss) * (softmax(z_m) - onehot(y_m)) / N    (0 for ignored m)
 * with N the number of valid tokens (0 <= y_m < V; y_m < 0 marks a token to
 * ignore; with no valid token the loss and dh are 0).  W (V x d) is frozen:
 * only dh is returned.  No bias.
 * How it runs: the forward is one tcgen05 GEMM over 256-token x 256-entry
 * tiles whose epilogue reduces each token's logits to a running (max, sum of
 * exp) per 128-entry block and picks up z[y]; no logit reaches memory.  Two
 * small kernels combine the blocks (log-sum-exp per token) and take the mean
 * in a fixed order.  The backward recomputes the logits chunk by chunk of
 * tokens, turns them into the bf16 gradient (softmax - onehot) * d(loss) / N
 * in the epilogue, and multiplies that chunk by W (K = V) for dh.
 * Conventions: H [M x d] bf16 and W [V x d] bf16 row-major, 16-byte aligned;
 * d % 8 == 0 and V % 8 == 0 (LORA_ERR_ALIGNMENT); labels int32 [M], lse fp32
 * [M], loss and dloss fp32 scalars, all device, 4-byte aligned.  A label >= V
 * sets status bit 0x2 and that token is ignored.
 * ------------------------------------------------------------------------ */
typedef struct lora_ce_desc {
    int64_t M;     /* tokens */
    int64_t d;     /* hidden size (features of h) */
    int64_t V;     /* vocabulary size (rows of W) */
} lora_ce_desc;

/* Bytes of device workspace lora_linear_ce_fwd (0), lora_linear_ce_bwd (1)
 * or lora_linear_ce_fwd_bwd (2) needs: the forward holds 8 bytes per token
 * and 128-entry block of the vocabulary plus 8 bytes per token; the backward
 * holds the gradient of the logits of one chunk of at most 8192 tokens
 * (chunk * V * 2 bytes); the fused call holds, per chunk, the forward's
 * partials, the chunk's fp32 logits and their bf16 gradient (chunk * V * 6
 * bytes, 6.3 GB at 8192 tokens and V = 128256).  The backward size is never
 * below the forward size.  0 for an invalid desc. */
size_t lora_linear_ce_workspace_size(const lora_ce_desc* desc, int for_backward);

/* Forward.  H, W (device, read); labels [M] (device, read); loss: device fp32
 * scalar (written: the mean over valid tokens); lse: device fp32 [M] (written:
 * each token's log-sum-exp, the backward's input).  M == 0 writes loss = 0 and
 * needs no H, labels or lse.  workspace >= lora_linear_ce_workspace_size(desc,
 * 0), 16-byte aligned (LORA_ERR_WORKSPACE); its header's status word as for
 * the layer.  Asynchronous on `stream`. */
lora_status_t lora_linear_ce_fwd(const lora_ce_desc* desc, const void* H, const void* W, const int32_t* labels,
                                 float* loss, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Backward: dH [M x d] bf16 (device, written) = d(loss) * dloss/dH with
 * *dloss (a device fp32 scalar, e.g. autograd's incoming gradient) as the
 * upstream factor.  lse: the forward's output.  Other arguments as the
 * forward; workspace >= lora_linear_ce_workspace_size(desc, 1). */
lora_status_t lora_linear_ce_bwd(const lora_ce_desc* desc, const void* H, const void* W, const int32_t* labels,
                                 const float* lse, const float* dloss, void* dH, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Forward and backward in one call, for a loss that is the step's final
 * scalar (its upstream factor *dloss already on the device, e.g. 1.0): the
 * fine-tuning libraries the pages describe compute this loss's gradient
 * during the forward pass, chunk by chunk.  Per chunk of at most 8192 tokens
 * the logit GEMM writes the chunk's fp32 logits to the workspace next to its
 * (max, sum) partials; the chunk's lse follows, then the logits' gradient
 * (bf16, the same arithmetic as lora_linear_ce_bwd) and dH = dz W.  The
 * logits are never recomputed, and never held beyond one chunk.  Writes loss,
 * lse and dH exactly as lora_linear_ce_fwd followed by lora_linear_ce_bwd
 * would (the same bits).  workspace >= lora_linear_ce_workspace_size(desc, 2);
 * other arguments and errors as those two calls. */
lora_status_t lora_linear_ce_fwd_bwd(const lora_ce_desc* desc, const void* H, const void* W, const int32_t* labels,
                                     const float* dloss, float* loss, float* lse, void* dH, void* workspace,
                                     size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_H */
