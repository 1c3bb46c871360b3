// Shared device helpers for the BasisKV sm_100a kernels: bulk copies into
// shared memory completed on mbarriers, bounded waits, bf16 tensor-core
// fragments, block scans.  Everything here is inline PTX or plain CUDA C++.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace basiskv {

constexpr uint32_t kStatusBadSlot = 1u;
constexpr uint32_t kStatusTimeout = 2u;
constexpr uint32_t kStatusBadPage = 4u;
constexpr uint32_t kStatusPartOverflow = 8u;  // a unit met more partials than it has slots
constexpr uint32_t kStatusBadLength = 16u;    // a length needs more pages than a table row holds
constexpr uint32_t kStatusDebugBounds = 32u;  // debug build: an index out of its range by construction

// Debug build (BASISKV_DEBUG): indices that the kernels keep in range by
// construction are checked where they are used; a failed check records
// kStatusDebugBounds and the access goes to index 0.  In the normal build the
// index passes through unchanged.
#ifdef BASISKV_DEBUG
__device__ __forceinline__ long long debug_index(long long i, long long bound, uint32_t* status) {
  if (i >= 0 && i < bound) return i;
  atomicOr(status, kStatusDebugBounds);
  return 0;
}
#define BASISKV_DEBUG_INDEX(i, bound, status) debug_index((i), (bound), (status))
#else
#define BASISKV_DEBUG_INDEX(i, bound, status) (i)
#endif

// Largest batch whose work plan travels in the kernel parameters; larger
// batches read the plan the prep grid writes to global memory.
constexpr int kPlanMax = 512;

// A bounded wait gives up after this many nanoseconds of %globaltimer.
#ifdef BASISKV_WAIT_TEST
// The wait-expiry test build: short waits, and the one copy that
// skip_issue_for_test names (item 1 of issuer 0: a warp of the per-warp-ring
// kernels, a CTA of the shared-ring one) is never issued, so its wait must
// run out.
constexpr uint64_t kWaitLimitNs = 1000000ull;
__device__ __forceinline__ bool skip_issue_for_test(int issuer, int item) {
  return issuer == 0 && item == 1;
}
#else
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool skip_issue_for_test(int, int) { return false; }
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// try_wait with a suspend-time hint: a waiting warp is descheduled (it does
// not compete for issue slots) until the phase completes or the hint runs out.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// On expiry sets kStatusTimeout and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

// Wait like mbar_wait, and also give up (without a status) once another
// warp of the CTA has set *abort; on expiry set both.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity, uint32_t* status,
                                                   volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// Atomic add with release and acquire semantics at gpu scope: the caller's
// earlier writes (and those ordered before them) are visible to whoever
// reads the new count, and the caller sees everything released by earlier
// adders.  Returns the old value.
__device__ __forceinline__ uint32_t atomic_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Arrive once on `bar` (release at CTA scope: the caller's earlier shared
// memory writes are visible to the thread that sees the phase complete).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// How long a routing warp waits for a folded query written by other warps
// before it folds the query itself.
constexpr uint64_t kFoldWaitNs = 50000ull;

// ---- bulk copy global -> shared (TMA unit, non-tensor form) -----------------
// dst, src 16-byte aligned, bytes a multiple of 16.  Completion is reported
// as transaction bytes on `bar`.  `policy` is an L2 cache policy descriptor.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// 8-byte relaxed (gpu scope) accesses: each is single-copy atomic, so a
// value and a tag packed into one word are seen together.
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t x;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(x) : "l"(p) : "memory");
  return x;
}
// Two consecutive words (p 16-byte aligned); each word is read atomically.
__device__ __forceinline__ void ld_relaxed_v2u64(const uint64_t* p, uint64_t& x, uint64_t& y) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(x), "=l"(y) : "l"(p) : "memory");
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

// ---- programmatic dependent launch ------------------------------------------
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---- shared-memory loads ----------------------------------------------------
__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}
__device__ __forceinline__ uint2 lds64(const void* p) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
  return v;
}
__device__ __forceinline__ uint32_t lds32(const void* p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)));
  return v;
}

// Four 8x8 bf16 matrices, transposed: lane l supplies the row address of
// matrix l/8, row l%8; register i receives matrix i in B-fragment order.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                              const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(row)));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& r0, uint32_t& r1, const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_addr(row)));
}

__device__ __forceinline__ void ldsm_x1_trans(uint32_t& r0, const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x1.trans.shared.b16 {%0}, [%1];" : "=r"(r0) : "r"(smem_addr(row)));
}

// ---- bf16 tensor-core MMA, fp32 accumulate ----------------------------------
// Register-only operations, so not volatile: the compiler may interleave
// independent accumulator chains.  The shared-memory loads that feed them
// stay volatile, in program order after the barrier waits.
// D(16x8) += A(16x16, row) * B(16x8, col)
__device__ __forceinline__ void mma_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D(16x8) += A(16x8, row) * B(8x8, col)
__device__ __forceinline__ void mma_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Pack two floats into a bf16x2 register (first argument in the low half).
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): a two-term split
// carrying ~16 significant bits, used where an fp32 operand meets bf16 data
// in the tensor cores.
__device__ __forceinline__ void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = __bfloat162float(__float2bfloat16_rn(x - hi));
}

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

// ---- warp / block reductions -------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan of one int per thread over a block of NT threads.  `tmp`
// holds NT/32 ints of shared memory.  Returns the exclusive prefix; *total
// receives the block sum.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  int base = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    int t = tmp[w];
    if (w < warp) base += t;
    sum += t;
  }
  __syncthreads();
  *total = sum;
  return base + x - v;
}

// Signal that this CTA finished its share of unit `u`; returns true in every
// thread of the one CTA that arrives last (which also resets the counter for
// the next call).  All global writes of the CTA made before the call are
// visible to the last CTA after it returns true.
__device__ __forceinline__ bool arrive_last(uint32_t* counter, uint32_t expected, int* flag_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(counter, 1u);
    const bool last = prev + 1 == expected;
    if (last) {
      *counter = 0u;
      __threadfence();
    }
    *flag_smem = last ? 1 : 0;
  }
  __syncthreads();
  return *flag_smem != 0;
}

}  // namespace basiskv
