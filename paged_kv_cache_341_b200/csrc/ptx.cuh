// sm_100a primitives used by the kernels: shared-memory mbarriers, TMA tile
// loads and bulk copies (each CTA loads its own tiles), a packed float32x2
// FMA, the base-2 exponential instruction, and bounded waits.
//
// Every wait is bounded in time: a wait that gives up sets the device error
// word (PA_DEVERR_TIMEOUT) and an abort flag in shared memory, so every other
// warp of the CTA stops waiting too and the kernel returns instead of hanging.
#ifndef PAGEDATTN_PTX_CUH
#define PAGEDATTN_PTX_CUH

#include <cuda.h>
#include <cstdint>

namespace pa {

// Device error word, read and cleared by pa_device_error().
__device__ int g_device_error;

enum DeviceError : int {
  DEVERR_BAD_BLOCK_ID = 1,   // block table entry outside [0, num_blocks)
  DEVERR_BAD_LENGTH = 2,     // context length beyond the block table (clamped)
  DEVERR_BAD_SLOT = 3,       // append slot outside the cache (skipped)
  DEVERR_BAD_PAIR = 4,       // copy pair id outside the pool (skipped)
  DEVERR_TIMEOUT = 5,        // a pipeline wait gave up (kernel returned early)
};

__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

// Upper bound for any single pipeline wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait until the phase of `bar` with parity `parity` has completed.  Returns
// false if the CTA aborted or the time limit passed (then the abort flag and
// the device error word are set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      set_device_error(DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Wait without honouring the abort flag (used while draining copies in flight
// before the CTA exits); still bounded in time.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      set_device_error(DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// L2 policy for data read exactly once (the K/V stream).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// L2 policy for data many CTAs read again soon (a shared prefix).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 3-D tile load global -> shared through a tensor map, completing on `bar`.
// The innermost coordinate c0 is always 0 here (16-byte aligned).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Contiguous bulk copy global -> shared (addresses 16-byte aligned, size a
// multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// d = a * b + d on a pair of float32 lanes (one instruction on sm_100a).
__device__ __forceinline__ void ffma2(float2& d, const float2 a, const float2 b) {
  asm("{\n\t.reg .b64 rd, ra, rb;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
}

// d += a on a pair of float32 lanes (one instruction on sm_100a).
__device__ __forceinline__ void fadd2(float2& d, const float2 a) {
  asm("{\n\t.reg .b64 rd, ra;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a.x), "f"(a.y));
}

// d = d * s on a pair of float32 lanes.
__device__ __forceinline__ void fmul2(float2& d, const float2 s) {
  asm("{\n\t.reg .b64 rd, rs;\n\t"
      "mov.b64 rs, {%2, %3};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "mul.rn.f32x2 rd, rd, rs;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(s.x), "f"(s.y));
}

// Programmatic dependent launch: let the next kernel on the stream launch now
// (its CTAs start and then wait), and, in that kernel, wait until the
// prerequisite grid has completed and its memory operations are visible.
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_prerequisite_grids() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 2^x with the hardware approximation (ex2.approx; 2^0 = 1 and 2^-inf = 0 exactly).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace pa

#endif
