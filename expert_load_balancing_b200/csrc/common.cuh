// common.cuh -- device helpers shared by the router kernels (sm_100a).
//
// Score order: every comparison of fp32 scores uses the order-preserving
// 32-bit key of the bit pattern (negative: all bits flipped; non-negative:
// sign bit set).  Keys compare as unsigned integers; equal keys are ties,
// broken toward the lower expert id.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kolibri_router.h"

namespace kolibri {

constexpr int kWarp = 32;

// Device status word.  Bit 0: a bounded wait expired; bit 1: a device-side
// argument check failed.  The library is built without relocatable device
// code, so every translation unit holds its own word (one per device);
// KOLIBRI_DEFINE_STATUS_TAKE gives each unit a host function that reads and
// clears it, and kolibri_device_status ORs them.
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadInput = 2u;
constexpr unsigned kStatusReadFailed = 0x80000000u;
static __device__ unsigned int g_status = 0u;

#define KOLIBRI_DEFINE_STATUS_TAKE(fn)                                              \
  unsigned fn() {                                                                   \
    unsigned v = 0u, zero = 0u;                                                     \
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess)               \
      return kStatusReadFailed;                                                     \
    if (v != 0u && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) \
      return kStatusReadFailed;                                                     \
    return v;                                                                       \
  }

__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_status, bits); }

__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t u = __float_as_uint(v);
  uint32_t s = static_cast<uint32_t>(static_cast<int32_t>(u) >> 31);  // 0 or ~0
  return u ^ (s | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// fp64 exp used by the gate.  Cody & Waite reduction x = k ln2 + r with ln2
// held as a double-double, degree-13 Taylor polynomial of e^r in Horner form
// with fused multiply-adds, then scaling by 2^k built in the exponent field.
// Only IEEE correctly rounded operations (explicit intrinsics, so the compiler
// cannot contract or reorder), valid for |x| <= 700.
__device__ __forceinline__ double gate_exp(double x) {
  const double kInvLn2 = 0x1.71547652b82fep+0;
  const double kLn2Hi = 0x1.62e42fefa39efp-1;
  const double kLn2Lo = 0x1.abc9e3b39803fp-56;
  double k = rint(__dmul_rn(x, kInvLn2));
  double r = __fma_rn(-k, kLn2Hi, x);
  r = __fma_rn(-k, kLn2Lo, r);
  double p = 0x1.6124613a86d09p-33;       // 1/13!
  p = __fma_rn(p, r, 0x1.1eed8eff8d898p-29);  // 1/12!
  p = __fma_rn(p, r, 0x1.ae64567f544e4p-26);  // 1/11!
  p = __fma_rn(p, r, 0x1.27e4fb7789f5cp-22);  // 1/10!
  p = __fma_rn(p, r, 0x1.71de3a556c734p-19);  // 1/9!
  p = __fma_rn(p, r, 0x1.a01a01a01a01ap-16);  // 1/8!
  p = __fma_rn(p, r, 0x1.a01a01a01a01ap-13);  // 1/7!
  p = __fma_rn(p, r, 0x1.6c16c16c16c17p-10);  // 1/6!
  p = __fma_rn(p, r, 0x1.1111111111111p-7);   // 1/5!
  p = __fma_rn(p, r, 0x1.5555555555555p-5);   // 1/4!
  p = __fma_rn(p, r, 0x1.5555555555555p-3);   // 1/3!
  p = __fma_rn(p, r, 0.5);                    // 1/2!
  p = __fma_rn(p, r, 1.0);                    // 1/1!
  p = __fma_rn(p, r, 1.0);                    // 1/0!
  long long ki = __double2ll_rn(k);
  double scale = __longlong_as_double((ki + 1023ll) << 52);
  return __dmul_rn(p, scale);
}

// Gate sigma(z) = 1 / (1 + e^-z) in fp64, rounded once to fp32.
__device__ __forceinline__ float gate_sigmoid(float z) {
  if (z > 700.0f) return 1.0f;
  if (z < -700.0f) return 0.0f;
  double t = gate_exp(-static_cast<double>(z));
  double s = __ddiv_rn(1.0, __dadd_rn(1.0, t));
  return __double2float_rn(s);
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

// One try: the thread may sleep in it until the phase completes, for at
// most about kSuspendNs, so waiting warps do not spin on issue slots.
constexpr uint32_t kSuspendNs = 200000u;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase.  Gives up after about `limit_ns`
// nanoseconds, records kStatusTimeout and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t start = global_timer_ns();
  while (true) {
    for (int i = 0; i < 4; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - start > limit_ns) {
      raise_status(kStatusTimeout);
      return false;
    }
  }
}

}  // namespace kolibri
