// Device helpers shared by the kernels of libmoe.so (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Bits of the device error word (first 4 bytes of the workspace).
constexpr uint32_t kErrTimeout = 1u;      // a bounded wait ran out
constexpr uint32_t kErrBadIndex = 2u;     // an index failed a kernel's own check

// Time limit of every device-side wait, in nanoseconds of %globaltimer: the
// workspace's control block holds it at byte kWaitLimitOffset (uint64,
// moe_workspace_set_wait_limit); 0 there means this default.  The drains
// after an abort always take the default.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr size_t kWaitLimitOffset = 8;

// The wait limit of the launch whose control block starts at `err` (read
// after pdl_wait: a copy before the launch may have set it).
__device__ __forceinline__ uint64_t wait_limit_ns(const uint32_t *err) {
  if (!err) return kWaitLimitNs;
  const uint64_t v = *reinterpret_cast<const volatile uint64_t *>(
      reinterpret_cast<const char *>(err) + kWaitLimitOffset);
  return v ? v : kWaitLimitNs;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialization (launch_kernel in moe_internal.h):
// it may become resident while the kernel before it on the stream is still
// running.  Each kernel therefore runs pdl_wait() in every thread before its
// first access to global memory (it returns once the previous kernel has
// completed and its writes are visible; at once when there is none), and no
// thread returns before it, so the completion of a kernel implies the
// completion of all kernels before it.  pdl_trigger() lets the next kernel
// start its own prologue early.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// bf16 <-> fp32
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);   // round to nearest even
  return *reinterpret_cast<uint32_t *>(&p);
}

// ---------------------------------------------------------------------------
// Fixed fp32 exponential for the softmax gate.
//
// Routing decisions that compare probabilities across tokens (expert choice,
// per-expert affinity dropping) must come out identically wherever the
// probabilities are evaluated, so exp is one fixed sequence of IEEE
// round-to-nearest fp32 operations with no fused multiply-add:
//   n = rint(z * log2 e)
//   r = (z - n * ln2_hi) - n * ln2_lo     (Cody-Waite; ln2_hi is ln 2
//                                           truncated to 16 bits, so n*ln2_hi
//                                           is exact for |n| < 256)
//   p = sum_{i=0..7} r^i / i!              (Taylor, Horner form, one rounded
//                                           multiply and one rounded add per
//                                           step)
//   exp(z) = p * 2^n                       (2^n from exponent bits)
// Valid for z <= 0 (the softmax argument after subtracting the row maximum);
// z < -87 returns 0.  The __f*_rn intrinsics are never contracted into FMAs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float exp_det(float z) {
  const float kLog2e = (float)1.4426950408889634;
  const float kLn2Hi = (float)(45426.0 / 65536.0);
  const float kLn2Lo = (float)(0.69314718055994530942 - 45426.0 / 65536.0);
  const float c0 = (float)(1.0), c1 = (float)(1.0), c2 = (float)(1.0 / 2.0),
              c3 = (float)(1.0 / 6.0), c4 = (float)(1.0 / 24.0), c5 = (float)(1.0 / 120.0),
              c6 = (float)(1.0 / 720.0), c7 = (float)(1.0 / 5040.0);
  float n = rintf(__fmul_rn(z, kLog2e));
  float r = __fsub_rn(z, __fmul_rn(n, kLn2Hi));
  r = __fsub_rn(r, __fmul_rn(n, kLn2Lo));
  float p = c7;
  p = __fadd_rn(__fmul_rn(p, r), c6);
  p = __fadd_rn(__fmul_rn(p, r), c5);
  p = __fadd_rn(__fmul_rn(p, r), c4);
  p = __fadd_rn(__fmul_rn(p, r), c3);
  p = __fadd_rn(__fmul_rn(p, r), c2);
  p = __fadd_rn(__fmul_rn(p, r), c1);
  p = __fadd_rn(__fmul_rn(p, r), c0);
  int ni = (int)n;
  ni = ni < -126 ? -126 : (ni > 0 ? 0 : ni);
  float scale = __int_as_float((ni + 127) << 23);
  float out = __fmul_rn(p, scale);
  return z < -87.0f ? 0.0f : out;
}

// SiLU(x) = x / (1 + e^-x) for the SwiGLU epilogues, with the fast
// reciprocal-based division (about 2 ulp in fp32; the results are rounded
// to bf16 next).  For x below about -88, e^-x is +inf and the quotient -0.
#ifndef MOE_FAST_SILU
#define MOE_FAST_SILU 1
#endif
__device__ __forceinline__ float silu_f(float x) {
  return MOE_FAST_SILU ? __fdividef(x, 1.0f + __expf(-x)) : x / (1.0f + __expf(-x));
}
// its sigmoid factor 1 / (1 + e^-x) (the SwiGLU derivative), the same way
__device__ __forceinline__ float sigmoid_f(float x) {
  return MOE_FAST_SILU ? __fdividef(1.0f, 1.0f + __expf(-x)) : 1.0f / (1.0f + __expf(-x));
}

// Composite selection key: larger probability first, then lower token.
__device__ __forceinline__ uint64_t affinity_key(float p, uint32_t t) {
  return ((uint64_t)__float_as_uint(p) << 32) | (uint64_t)(0xffffffffu - t);
}

}  // namespace moe
