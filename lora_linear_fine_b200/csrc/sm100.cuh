// sm100.cuh — thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// LoRA-linear kernels use: mbarriers with bounded waits, TMA tiled loads,
// tcgen05 (TMEM allocation, MMA issue, commit, loads) and the shared-memory /
// instruction descriptors of tcgen05.mma kind::f16.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace lora {

constexpr int kSmemLimitBytes = 232448;  // max dynamic shared memory per block on sm_100

// ----------------------------------------------------------------------------
// device status word (lives at offset 0 of the caller's workspace)
// ----------------------------------------------------------------------------
enum : uint32_t {
  kStatusWaitTimeout = 0x1u,   // a bounded mbarrier wait gave up
  kStatusBadArgument = 0x2u,   // a device-side argument check failed
  kStatusF16Range = 0x4u,      // a value converted to fp16 was outside its finite range
};

// A wait gives up after this many SM clock cycles (several seconds at any
// clock the part runs at); legitimate waits last microseconds.
constexpr long long kWaitLimitCycles = 1ll << 34;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t elect_lane0() { return (threadIdx.x & 31u) == 0u; }

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Shared abort state of one CTA: once any waiter gives up, every other wait
// in the CTA returns false promptly so all warps reach the common teardown.
struct AbortCtl {
  volatile uint32_t* flag;     // in shared memory
  uint32_t* status;            // device status word (global), may be null
};

// Wait for the phase with parity `parity` of `bar` to complete.  Returns false
// if the CTA is aborting or the wait exceeded kWaitLimitCycles (then the status
// word and the CTA abort flag are set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const AbortCtl& ctl,
                                          long long limit_cycles = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*ctl.flag) return false;
    if (clock64() - t0 > limit_cycles) {
      if (ctl.status) atomicOr(ctl.status, kStatusWaitTimeout);
      *ctl.flag = 1u;
      return false;
    }
  }
}

// Position in a ring of pipeline stages: slot index and the parity of its
// current mbarrier phase.
struct RingPos {
  uint32_t stage = 0, phase = 0;
  __device__ __forceinline__ void next(int stages) {
    if (++stage == static_cast<uint32_t>(stages)) { stage = 0; phase ^= 1u; }
  }
};

// ----------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion on an mbarrier)
// ----------------------------------------------------------------------------
// Untiled bulk copy of `bytes` contiguous bytes global -> this CTA's shared
// memory, completion counted on `bar` (both addresses 16-byte aligned, bytes a
// multiple of 16).
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// 2D tiled load of the box at coordinates (x = inner, y = outer).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Same, with an L2 eviction-priority hint (createpolicy result).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* tm, uint64_t* bar, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// 3D tiled load of the box at coordinates (x, y, z), with an L2 eviction
// hint (createpolicy result) or without (policy 0 is not a valid policy, so
// two forms).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* tm, uint64_t* bar, int32_t x,
                                                 int32_t y, int32_t z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte global store that does not allocate in L1 and carries an L2
// eviction-priority policy (outputs written once: evict first).
__device__ __forceinline__ void st_global_v4_hint(void* ptr, uint4 v, uint64_t policy) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy)
               : "memory");
}

// Named barrier `id` over `n` threads that also ANDs a predicate: every
// participant gets the same answer, so a group can leave a loop together
// when any of its bounded waits gave up.
template <int id, int n>
__device__ __forceinline__ bool bar_sync_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(id), "n"(n)
      : "memory");
  return r != 0u;
}

template <int id, int n>
__device__ __forceinline__ void bar_sync_named() {
  asm volatile("barrier.cta.sync %0, %1;" ::"n"(id), "n"(n) : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while its predecessor in the stream is finishing;
// grid_dep_wait() blocks the calling thread until the predecessor grid has
// completed and its memory operations are visible (without the attribute it
// returns at once).  Every kernel here calls it from every thread after its
// prologue (barriers, tensor memory) and before its first global access.
// Right after the wait it lets the next kernel in the stream be launched
// (griddepcontrol.launch_dependents): that kernel's CTAs are placed as SMs
// free up and run their own prologue while this grid finishes; they touch
// global memory only after their own wait, i.e. after this grid completed.
// Triggering after the wait keeps at most one grid launched ahead.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy
// (tensor core operand reads, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA tiled store of one box from this CTA's shared memory to global memory,
// tracked in the thread's bulk async-group (commit, then wait).  Coordinates
// are non-negative; the tensor map's bounds clip a box that runs past the
// tensor's last row or column.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* tm, const void* src, int32_t x, int32_t y,
                                                  uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(tm),
      "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
// The same box added element by element to what global memory holds (the
// addition is done at L2; fp32 tensor maps).
__device__ __forceinline__ void tma_reduce_add_2d_hint(const CUtensorMap* tm, const void* src, int32_t x, int32_t y,
                                                       uint64_t policy) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
      ::"l"(tm), "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The same between generic-proxy global accesses and TMA (async-proxy)
// accesses of global memory: a CTA that publishes data with plain stores for
// another CTA's TMA loads fences after its stores, and the reader fences
// after it has acquired the flag and before it issues the loads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Publication flags in global memory: OR with release semantics at GPU scope
// (the writer's earlier stores become visible to any thread that acquires
// the bit), and a load with acquire semantics.
__device__ __forceinline__ void red_or_release_gpu(uint32_t* addr, uint32_t bits) {
  asm volatile("red.release.gpu.global.or.b32 [%0], %1;" ::"l"(addr), "r"(bits) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* addr) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

// Wait until all of `bits` are set in the global word at addr (set by
// another CTA of the same grid).  Bounded like mbar_wait: gives up after
// kWaitLimitCycles, sets the status word and the CTA's abort flag, and
// returns false; returns false at once if the CTA is already aborting.
__device__ __forceinline__ bool flag_wait_all(const uint32_t* addr, uint32_t bits, const AbortCtl& ctl) {
  if ((ld_acquire_gpu(addr) & bits) == bits) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(64);
    if ((ld_acquire_gpu(addr) & bits) == bits) return true;
    if (*ctl.flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      if (ctl.status) atomicOr(ctl.status, kStatusWaitTimeout);
      *ctl.flag = 1u;
      return false;
    }
  }
}

// ----------------------------------------------------------------------------
// Dropout keep bits: one bit per element, bit j of byte b keeping element
// 8 b + j of a row of `ld` bytes.
// ----------------------------------------------------------------------------

// kBytes consecutive keep bytes of one row from byte b0 (a multiple of
// kBytes), packed four to a word.  One vector load when the row start is
// kBytes-aligned (`vec`), byte loads otherwise; bytes at or past `ld`, and all
// bytes of a row that does not exist (!ok), read as 0.  All loads are issued
// before any value is used, so their latencies overlap.
template <int kBytes>
__device__ __forceinline__ void load_keep_bytes(const uint8_t* mrow, int b0, int ld, bool ok, bool vec,
                                                uint32_t (&m)[kBytes / 4]) {
  static_assert(kBytes == 8 || kBytes == 16, "8 or 16 keep bytes");
  if (ok && vec && b0 + kBytes <= ld) {
    if constexpr (kBytes == 16) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(mrow + b0));
      m[0] = v.x; m[1] = v.y; m[2] = v.z; m[3] = v.w;
    } else {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(mrow + b0));
      m[0] = v.x; m[1] = v.y;
    }
    return;
  }
  uint32_t b[kBytes];
#pragma unroll
  for (int c = 0; c < kBytes; ++c) b[c] = (ok && b0 + c < ld) ? static_cast<uint32_t>(__ldg(mrow + b0 + c)) : 0u;
#pragma unroll
  for (int w = 0; w < kBytes / 4; ++w) m[w] = b[4 * w] | (b[4 * w + 1] << 8) | (b[4 * w + 2] << 16) | (b[4 * w + 3] << 24);
}

// Zero the dropped elements of one 128-byte row in each of kBoxes
// SWIZZLE_128B bf16 boxes (box k at row_base + k * box_stride): 16-byte chunk
// c (elements 8c .. 8c + 7) of box k sits at position c ^ (row & 7) and takes
// keep byte 8k + c (byte (8k + c) % 4 of word (8k + c) / 4 of `m`).  All
// chunks are read before any is written, so the row costs one shared-memory
// latency.
template <int kBoxes>
__device__ __forceinline__ void mask_sw128_rows(uint8_t* row_base, int box_stride, int row, const uint32_t* m) {
  uint4 v[kBoxes][8];
#pragma unroll
  for (int k = 0; k < kBoxes; ++k)
#pragma unroll
    for (int c = 0; c < 8; ++c) v[k][c] = reinterpret_cast<const uint4*>(row_base + k * box_stride)[c ^ (row & 7)];
#pragma unroll
  for (int k = 0; k < kBoxes; ++k) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = 8 * k + c;
      const uint32_t b = (m[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      if (b == 0xFFu) continue;
      const uint32_t w[4] = {v[k][c].x, v[k][c].y, v[k][c].z, v[k][c].w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = (b >> (2 * e)) & 1u ? 0x0000FFFFu : 0u;
        const uint32_t hi = (b >> (2 * e + 1)) & 1u ? 0xFFFF0000u : 0u;
        o[e] = w[e] & (lo | hi);
      }
      reinterpret_cast<uint4*>(row_base + k * box_stride)[c ^ (row & 7)] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA
// ----------------------------------------------------------------------------
// Allocate `ncols` (power of two >= 32) TMEM columns; the base address is
// written to *dst_smem.  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate.  Issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes: thread i gets
// lane (base lane + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// 16 columns variant.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15])
      : "r"(taddr));
}

// Store 16 consecutive 32-bit columns to this warp's 32 TMEM lanes (lane i of
// the warp writes lane (lane field of taddr) + i); tmem_wait_st() makes the
// warp's stores complete.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------------------------------
// descriptors
// ----------------------------------------------------------------------------
// Shared-memory matrix descriptor for the 128-byte swizzled canonical layouts
// (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B; tiles 1024-B aligned):
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4
//   bits 32-45  stride-dimension byte offset >> 4
//   bits 46-47  descriptor version (1 on sm_100)
//   bits 61-63  layout: 2 = SWIZZLE_128B
// K-major operand: rows of 128 B (64 bf16 along K), 8-row groups `sbo` apart;
//   `lbo` is unused (set to 16 B).  A K step of 16 elements inside the 128-B
//   row is a +32 B change of the start address.
// MN-major operand: rows of 128 B hold 64 consecutive M/N elements for one K;
//   8 K-rows form a 1024-B atom; `sbo` = distance between 8-row K groups,
//   `lbo` = distance between 64-element M/N blocks.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with fp32 D:
//   bits 4-5 D format (1 = f32), 7-9 A format, 10-12 B format (0 = f16, 1 = bf16;
//   A and B always share one type here), bit 15 A major (1 = MN-major), bit 16
//   B major, bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_mma(int m, int n, bool a_mn_major, bool b_mn_major, bool f16) {
  return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) |
         (static_cast<uint32_t>(a_mn_major) << 15) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn_major, bool b_mn_major) {
  return idesc_mma(m, n, a_mn_major, b_mn_major, false);
}

// Byte offset of element (row, col) (bf16) inside a K-major SWIZZLE_128B tile
// whose rows are 128 B (64 elements) and whose base is 1024-B aligned: the
// 16-byte chunk index is XORed with (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col) {
  const uint32_t chunk = (col >> 3) ^ (row & 7u);
  return (row >> 3) * 1024u + (row & 7u) * 128u + chunk * 16u + (col & 7u) * 2u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ----------------------------------------------------------------------------
// CTA pairs (thread-block cluster of 2) and tcgen05 cta_group::2
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of any CTA in the cluster (address from mapa_shared).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Parity wait with cluster-scope acquire (the phase may be completed by a peer CTA).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, const AbortCtl& ctl) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*ctl.flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      if (ctl.status) atomicOr(ctl.status, kStatusWaitTimeout);
      *ctl.flag = 1u;
      return false;
    }
  }
}

// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar_cluster` from mapa_shared).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, uint32_t bar_cluster, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A * B over the CTA pair: M = 256 (128 rows in each CTA's tensor memory),
// A and B halves read from each CTA's shared memory at the same offsets.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at the same offset in every CTA of `cta_mask`
// when the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

}  // namespace lora
