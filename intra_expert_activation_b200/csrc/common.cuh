// Device helpers shared by the sm_100a kernels: mbarriers with bounded
// waits, TMA tensor loads, tcgen05 (TMEM alloc / MMA / commit / load) and
// the shared-memory and instruction descriptors of kind::f16 MMAs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------- status

// Record a device-side error in the status word (first error wins).
__device__ __forceinline__ void report_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Checked builds (-DMOE_CHECK=1, `build.py --check`): bounds checks on the
// indices the kernels compute from data (slots, union rows). A failed check
// records MOE_ERR_INVALID in the status word and the caller skips or clamps
// the access; in the normal build the checks compile away.
#ifndef MOE_CHECK
#define MOE_CHECK 0
#endif
__device__ __forceinline__ bool moe_in_bounds(int* status, bool ok) {
  if (MOE_CHECK && !ok) {
    report_error(status, kErrDeviceInvalid);
    return false;
  }
  return true;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }

// Wait until the previous kernel on the stream has completed and its memory is
// visible (no-op when the launch had no programmatic dependency). Every CTA
// calls it before it exits, so a grid completes only after its predecessor
// has. No explicit early trigger: the next kernel's launch starts as this
// grid's CTAs exit. (An explicit `griddepcontrol.launch_dependents` at entry
// let the next kernel's CTAs take SM slots while this one ran, and the
// layer measured 2-7 us slower per batch on the Mixtral-shaped decode.)
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
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
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up after
// about a second (limit probes; the kernels keep the default, the checked
// build's timeout test passes a small one): sets *abort, records
// MOE_ERR_DEVICE_TIMEOUT and returns false, so that no kernel can hang the
// GPU on a lost arrival.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status, int tight = 0,
                                          uint32_t limit = kSpinLimit) {
  // optionally first a tight run of probes (each may suspend the thread
  // briefly in hardware), for waits that are short and on the critical path;
  // then probes with growing sleeps up to the limit
  for (int i = 0; i < tight; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  if (mbar_try_wait(bar, parity)) return true;
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    __nanosleep(i < 64 ? 20 : 200);
  }
  *abort = 1;
  report_error(status, kErrDeviceTimeout);
  return false;
}

// One lane of the warp waits; the outcome is broadcast, so the warp never
// diverges around a later __syncwarp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status, int tight = 0,
                                          uint32_t limit = kSpinLimit) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status, tight, limit) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait for another CTA's release flag (acquire), at most limit
// probes (about a second by default); on expiry as mbar_wait.
__device__ __forceinline__ bool wait_flag(const int* f, volatile int* abort, int* status,
                                          uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < limit; ++i) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v) return true;
    if (*abort) return false;
    __nanosleep(i < 64 ? 20 : 200);
  }
  *abort = 1;
  report_error(status, kErrDeviceTimeout);
  return false;
}

// ---------------------------------------------------------------- TMA

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completion counted on bar as
// transaction bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled tensor load into this CTA's shared memory; completion is
// signalled to bar as transaction bytes. x is the inner (contiguous)
// coordinate; every caller passes x as a multiple of 64 elements (128 B).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Same with an L2 eviction-priority hint (streamed weights: evict first).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map,
                                                 uint64_t* bar, int32_t x, int32_t y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tcgen05

// Allocate ncols TMEM columns (power of two >= 32); the base address is
// written to *dst in shared memory. Executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate; one thread issues.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on bar when every MMA issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i gets row (lane base + i).
// The registers are valid only after tmem_ld_wait(r...) below, which takes
// them as in/out operands so that no use can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld_wait(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]),
                 "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]),
                 "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(b[0]), "+r"(b[1]),
                 "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                 "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]),
                 "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}

// Shared-memory matrix descriptor for a tcgen05 operand tile laid out in
// the canonical 128-byte-swizzle form (1024-byte aligned atoms of 8 rows x
// 128 bytes). lbo/sbo are byte offsets:
//  K-major tiles: rows of 128 B along K; sbo = 1024 (next 8 rows), lbo unused.
//  MN-major tiles: 64 MN-elements (128 B) per K-row; lbo = offset of the next
//  64-element MN atom, sbo = offset of the next group of 8 K-rows.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for tcgen05
  d |= 2ull << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, dense.
// a_mn / b_mn: 1 if that operand is MN-major in shared memory.
__host__ __device__ __forceinline__ uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, uint32_t a_mn,
                                                            uint32_t b_mn) {
  uint32_t d = 0;
  d |= 1u << 4;          // D format: f32
  d |= 1u << 7;          // A format: bf16
  d |= 1u << 10;         // B format: bf16
  d |= (a_mn & 1u) << 15;
  d |= (b_mn & 1u) << 16;
  d |= ((N >> 3) & 0x3Fu) << 17;
  d |= ((M >> 4) & 0x1Fu) << 24;
  return d;
}

// ---------------------------------------------------------------- direct combine

// Under Dims::direct_combine the row stream adds w x the sums of a slot straight
// into its token's output accumulator row Y[token] (zeroed by the router), and
// the last CTA of the last kernel that adds writes out from those rows.

// The output row and combine weight of slot s (routed: the token the router
// placed there and its weight; shared: weight 1).
__device__ __forceinline__ void slot_target(const Dims& dm, const Workspace& ws, int s, int& tok,
                                            float& w) {
  if (s < dm.slots_routed) {
    tok = __ldcg(ws.perm + s);
    w = __ldcg(ws.slot_w + s);
  } else {
    tok = (s - dm.slots_routed) % dm.T_pad;
    w = 1.f;
  }
  if (!moe_in_bounds(ws.status, tok >= 0 && tok < dm.T)) tok = 0;  // checked build
}

// Direct combine, every thread of every CTA: after this CTA's sums are out,
// take the ticket; the last CTA writes out[t][c] = Y[t][c] for t < T.
static __device__ void direct_finish(const Dims& dm, const Workspace& ws, void* out, int out_bf16) {
  __shared__ int is_last;
  __threadfence();  // this thread's sums are visible before the ticket
  __syncthreads();
  if (threadIdx.x == 0)
    is_last = atomicAdd(ws.meta + kMetaDownDone, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) {  // every CTA has its ticket: ready for the next forward
    ws.meta[kMetaDownDone] = 0;
    ws.meta[kMetaRoute1] = 0;
  }
  const int n4 = dm.T * dm.d / 4;
  const float4* y4 = reinterpret_cast<const float4*>(ws.y);
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = __ldcg(y4 + i);
    if (out_bf16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&lo);
      u.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(out)[i] = u;
    } else {
      reinterpret_cast<float4*>(out)[i] = v;
    }
  }
}

// ---------------------------------------------------------------- misc

// Vector fp32 atomic adds (no return value) into global memory.
__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// 16 bytes of read-only data that is read once: not kept in L1. Not
// volatile, so the compiler may schedule it (callers issue several
// unconditionally before the first use; a load under a branch would be
// waited for at the branch's join).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// SiLU(g) = g / (1 + e^-g) with the fast exponential and division intrinsics
// (a few ulp of fp32; the threshold band is 1e-3 of tau). For g below about
// -88, e^-g overflows to +inf and the quotient is -0.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

}  // namespace moe
