// Shared device helpers of libhga: element traits, exact rounding, the device
// status word and small warp utilities.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hga.h"

namespace hga {

// Device status word: kernels record HGA_ERR_DEVICE_CHECK / HGA_ERR_TIMEOUT
// here instead of trapping; hga_check() reads and clears it.
__device__ int g_status;

__device__ __forceinline__ void report(int code) { atomicCAS(&g_status, 0, code); }

// Limit of every bounded wait of the tensor-core kernels, in nanoseconds
// (2 s unless hga_set_wait_limit_ns changed it for the device).
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

// Programmatic dependent launch: every kernel of the library is launched so
// that it may start while the previous kernel of the stream is finishing;
// griddep_wait() blocks until that kernel has completed and its writes are
// visible (call it before reading any input), griddep_launch() lets the next
// kernel start launching (called once a CTA's main work is done).  Both are
// no-ops without the launch attribute.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---------------------------------------------------------------- rounding

// float64 -> bfloat16, round to nearest even, in one rounding: round to odd
// into float32 (24 bits >= 8 + 2, so no double-rounding error), then round to
// nearest even into bfloat16 (Boldo & Melquiond, "Emulation of FMA and
// correctly rounded sums: proved algorithms using rounding to odd", 2008).
__device__ __forceinline__ __nv_bfloat16 f64_to_bf16_rne(double x) {
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __float2bfloat16_rn(f);
}

template <typename T> struct Elt;
template <> struct Elt<__nv_bfloat16> {
  static constexpr int kVec = 8;  // elements per 16-byte load
  __device__ static __forceinline__ void widen(const uint4& raw, double* out) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ static __forceinline__ __nv_bfloat16 from_f64(double x) { return f64_to_bf16_rne(x); }
  __device__ static __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Elt<float> {
  static constexpr int kVec = 4;
  __device__ static __forceinline__ void widen(const uint4& raw, double* out) {
    const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = f[i];
  }
  __device__ static __forceinline__ float from_f64(double x) { return __double2float_rn(x); }
  __device__ static __forceinline__ float to_f32(float x) { return x; }
  __device__ static __forceinline__ float from_f32(float x) { return x; }
};

// Order-preserving map of a float score to an unsigned key (larger score ->
// larger key); -0 is folded onto +0 so that equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

}  // namespace hga
