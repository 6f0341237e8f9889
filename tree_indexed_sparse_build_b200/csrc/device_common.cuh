// Device helpers shared by the sm_100a kernels: dtype loads, warp reductions,
// mbarrier and bulk-copy (1-D TMA) wrappers.  No cluster multicast anywhere.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace zha {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Round-to-nearest-even fp32 -> bf16 bits (finite inputs; NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Unpack 16 bytes of storage into fp32: 8 bf16 or 4 fp32 values.
template <typename T> struct Vec16;
template <> struct Vec16<uint16_t> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void to_f32(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
    o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
    o[4] = __uint_as_float(v.z << 16); o[5] = __uint_as_float(v.z & 0xFFFF0000u);
    o[6] = __uint_as_float(v.w << 16); o[7] = __uint_as_float(v.w & 0xFFFF0000u);
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void to_f32(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
  }
};

// Summary storage (fp32, or bf16 bits in uint16_t).  store(): the stored element of a node
// whose fp64 mean is v (nearest fp32; for bf16 that fp32 rounded once more to the nearest
// bf16, ties to even).  kept(): the fp64 value the node's parent averages -- for bf16 the
// stored value itself; fp32 trees keep the unrounded fp64 mean between the levels that one
// kernel computes.  load(): a stored element as fp32.
template <typename TS> struct SumT;
template <> struct SumT<float> {
  __device__ __forceinline__ static float store(double v) { return __double2float_rn(v); }
  __device__ __forceinline__ static double kept(double v) { return v; }
  __device__ __forceinline__ static float load(float x) { return x; }
};
template <> struct SumT<uint16_t> {
  __device__ __forceinline__ static uint16_t store(double v) { return f32_to_bf16_bits(__double2float_rn(v)); }
  __device__ __forceinline__ static double kept(double v) { return (double)bf16_bits_to_f32(store(v)); }
  __device__ __forceinline__ static float load(uint16_t x) { return bf16_bits_to_f32(x); }
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

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

// ---- mbarrier + bulk copy (non-multicast 1-D TMA) ---------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Ends the life of an mbarrier object, so its shared memory may hold other data (bulk
// copies included).  Every thread must be done with it.
__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) accesses of the same CTA's shared memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One arrival on `bar` (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
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
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Global -> shared bulk copy completing on `bar`.  dst, src 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Non-blocking test of phase `parity` of `bar` (no suspension).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounds below this many SM clocks (set only to test the failure path) poll with test_wait:
// try_wait suspends the thread until the phase completes or a hardware time limit passes, so
// a tiny bound would never be noticed before the copies land.
constexpr long long kPollWaitBelow = 1000000;

// Bounded wait on phase `parity` of `bar`.  Gives up after ~max_cycles SM clocks,
// records kDevErrTimeout-style `flag` in *err and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned* err,
                                                  unsigned flag, long long max_cycles) {
  if (max_cycles < kPollWaitBelow) {
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity)) {
      if (clock64() - t0 > max_cycles) {
        atomicOr(err, flag);
        return false;
      }
    }
    return true;
  }
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > max_cycles) {
      atomicOr(err, flag);
      return false;
    }
  }
  return true;
}

}  // namespace zha

namespace zha {

// Named CTA barriers over a group of warps: barrier `id` (1..15) with `nthreads` threads (a
// multiple of 32, every thread of the group arrives).  Used when several queries share a
// CTA and each query owns a group of warps.
__device__ __forceinline__ void group_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Number of threads of the group with p true (a barrier as well).
__device__ __forceinline__ int group_count(int id, int nthreads, bool p) {
  int r;
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.popc.u32 %0, %2, %3, q;\n\t}"
      : "=r"(r)
      : "r"((int)p), "r"(id), "r"(nthreads)
      : "memory");
  return r;
}
// True if p holds for any thread of the group (a barrier as well).
__device__ __forceinline__ bool group_any(int id, int nthreads, bool p) {
  int r;
  asm volatile(
      "{\n\t.reg .pred q, o;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred o, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}"
      : "=r"(r)
      : "r"((int)p), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still running;
// pdl_wait() blocks until that kernel has completed and its writes are visible, so it
// must precede the first read of anything an earlier kernel produced.
// pdl_release() lets the next kernel in the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace zha
