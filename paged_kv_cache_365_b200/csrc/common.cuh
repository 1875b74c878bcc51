// Shared device helpers: storage formats, 16-byte chunk conversions, the
// device error word, and hand-written PTX for the mbarrier / bulk-copy
// staging pipeline (sm_90+ instructions, used here on sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

constexpr int kBlockSize = PKV_BLOCK_SIZE;

// Device error word (PKV_ERR_* bits), one per device; read and cleared by
// pkv_get_error.  Defined here: the library is a single translation unit of
// device code (pkv_api.cu), which is the only file that includes this one.
__device__ unsigned int g_error_word = 0u;

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

// Programmatic dependent launch.  Every library kernel is launched with
// programmatic stream serialization, so it may be scheduled while the
// previous kernel in the stream is still draining.  Each kernel calls
// pdl_wait() before its first global-memory access (that makes the previous
// kernel's writes visible, whatever that kernel was), then pdl_trigger() so
// that the next kernel can be scheduled once every CTA of this one started.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

// 2^x for the online softmax: the SFU's approximate base-2 exponential
// (PTX ex2.approx.ftz.f32: a few ulp; results below 2^-126 flush to zero, a
// weight no sum can notice next to the running max's 2^0; 2^-inf = 0).
__device__ __forceinline__ float exp2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// storage formats: a 16-byte chunk holds kVec elements
// ---------------------------------------------------------------------------
template <typename T>
struct Fmt;

template <>
struct Fmt<float> {
  static constexpr int kVec = 4;
  __device__ __forceinline__ static void to_f32(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ static float from_f32(float x) { return x; }
};

template <>
struct Fmt<__half> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static void to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 t = __half22float2(h);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ __forceinline__ static __half from_f32(float x) { return __float2half_rn(x); }
};

template <>
struct Fmt<__nv_bfloat16> {
  static constexpr int kVec = 8;
  // a bf16 value is the upper half of a float32: widening is a shift/mask
  __device__ __forceinline__ static void to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// ---------------------------------------------------------------------------
// shared-memory access and the async staging pipeline
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// make barrier initialisation visible to the async proxy (bulk copies)
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// order this thread's earlier generic-proxy shared accesses before later
// async-proxy (bulk copy) accesses to the same memory
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Non-blocking test: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of a barrier, giving up after ~`limit_cycles`
// SM clocks.  Returns false on give-up (the caller flags PKV_ERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  long long limit_cycles = (1ll << 32)) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit_cycles) return false;
  }
  return true;
}

// Bulk (non-tensor) copy global -> this CTA's shared memory, completing
// `bytes` of transaction count on `bar`.  src, dst 16-byte aligned; bytes a
// multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ float warp_max(float v, int from_mask = 16, int to_mask = 1) {
  for (int m = from_mask; m >= to_mask; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

}  // namespace pkv
