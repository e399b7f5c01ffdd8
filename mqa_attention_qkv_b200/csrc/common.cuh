// Device helpers shared by the kernels of libgqa_b200: storage conversion,
// the device error word, and the bounded waits every pipeline uses.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gqa.h"

namespace gqa {

// ---------------------------------------------------------------------------
// storage type <-> float
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// ---------------------------------------------------------------------------
// device error word (bits of gqa_device_error_bits)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// ---------------------------------------------------------------------------
// Rotary embedding angle.  inv_freq_i = theta^(-2i/hd) and the angle
// position * inv_freq_i are formed in double precision and reduced to
// [-pi, pi] before the float sincos, so the angle error stays ~1e-7 rad even
// at position 8191 (a float product would carry ~5e-4 rad there).  On that
// reduced range the hardware approximation __sincosf is accurate to about
// 2^-21 absolute, far below a bf16 output's rounding, and takes two MUFU
// operations instead of the ~40 instructions of the full-range sincosf: in
// the projection GEMM's epilogue the full-range call measured as ~20% of the
// whole kernel.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double rope_inv_freq(int i, int hd, double theta) {
  return pow(theta, -2.0 * (double)i / (double)hd);
}

__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = (double)pos * inv_freq;
  a -= two_pi * rint(a * (1.0 / two_pi));
  __sincosf((float)a, s, c);
}

// The same angle in fixed point, for loops that evaluate many angles: the
// angle in turns, pos * inv_freq / (2 pi), modulo 1 in 0.64 fixed point.
// step = frac(inv_freq / (2 pi)) * 2^64 is formed once in double (relative
// error 2^-53); the product with the sign-extended position wraps modulo
// 2^64, which is exactly the reduction modulo 2 pi, and the top 32 bits read
// as a signed integer are the angle in [-1/2, 1/2) turns.  Integer multiplies
// replace the five double-precision operations of rope_cos_sin; the angle
// error stays below 2e-7 rad at any position.
__device__ __forceinline__ unsigned long long rope_turn_step(double inv_freq) {
  double turns = inv_freq * (1.0 / 6.283185307179586476925286766559);
  turns -= floor(turns);
  return (unsigned long long)fmin(turns * 18446744073709551616.0, 18446744073709549568.0);
}

__device__ __forceinline__ void rope_cos_sin_fx(int pos, unsigned long long step, float* c, float* s) {
  const unsigned long long t = (unsigned long long)(long long)pos * step;
  const float a = (float)(int)(t >> 32) * 1.46291807926715968e-9f;   // 2 pi / 2^32
  __sincosf(a, s, c);
}

// ---------------------------------------------------------------------------
// Time-bounded waits.  A wait that has not succeeded after its limit gives
// up, records GQA_DEVERR_WAIT_TIMEOUT and returns false; the caller then skips
// the rest of its work and goes straight to its teardown.  The limit is
// kWaitLimitNs unless the device error word's companion (words 2-3 of the
// 16-byte block `err` points at) holds a shorter one, which the failure-path
// tests set through gqa_debug_set_wait_limit_ns.
// ---------------------------------------------------------------------------
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t wait_limit_ns(const int* err) {
  const uint64_t v = err ? *reinterpret_cast<const volatile uint64_t*>(err + 2) : 0ull;
  return v ? v : kWaitLimitNs;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may start while the kernel before it in the
// stream is still running: it must wait (pdl_wait) before its first access to
// global memory that the earlier kernel may write or read, after which all of
// that kernel's writes are visible.  Without such a predecessor both are
// no-ops.  pdl_launch_dependents lets the next kernel in the stream launch as
// soon as every CTA of this one has issued it (that kernel waits in its turn).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier to complete; bounded in time.  Once
// any wait has given up (the timeout bit of the error word is set), every
// other wait gives up at its next check too, so a broken pipeline ends the
// whole grid within about one limit instead of one limit per CTA.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint64_t limit = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (err && (*reinterpret_cast<volatile int*>(err) & GQA_DEVERR_WAIT_TIMEOUT)) return false;
      if (!limit) limit = wait_limit_ns(err);
      if (global_timer_ns() - t0 > limit) {
        raise_error(err, GQA_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Teardown wait for work this thread itself issued (copies or MMAs in
// flight), which completes on its own: bounded by the limit alone, not cut
// short when another wait has already given up, so that a role that stops
// early still lets its asynchronous work land before shared memory or TMEM
// is released.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, int* err) {
  const uint64_t t0 = global_timer_ns();
  uint64_t limit = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (!limit) limit = wait_limit_ns(err);
      if (global_timer_ns() - t0 > limit) {
        raise_error(err, GQA_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

}  // namespace gqa
