// Shared device helpers of the B200 Star / Pulsar attention library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/pulsar.h"

namespace pa {

// First 256 bytes of every workspace: the device status block.
struct DeviceStatus {
  int32_t code;    // 0 or a negative pa_status; first error wins
  int32_t info0;   // kernel-specific detail (e.g. offending index)
  int32_t info1;
  int32_t pad[61];
};
static_assert(sizeof(DeviceStatus) == 256, "status block is 256 bytes");

constexpr size_t kStatusBytes = 256;
constexpr size_t kAlign = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a = kAlign) {
  return (x + a - 1) / a * a;
}

__device__ inline void set_status(DeviceStatus* st, int code, int info0 = 0, int info1 = 0) {
  if (st == nullptr) return;
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->info0 = info0;
    st->info1 = info1;
  }
}

// ln(2) and log2(e) in fp32/fp64.
constexpr float kLn2f = 0.693147180559945309417f;
constexpr double kLog2e = 1.44269504088896340736;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// Load with L2-only caching (values other SMs update with atomics).
__device__ __forceinline__ unsigned long long ld_cg_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return v;
}

}  // namespace pa
