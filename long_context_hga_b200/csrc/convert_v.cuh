// V storage in fp16 for the attention kernels' P.V product.
//
// The attention keeps P in fp16 (11 significant bits); tcgen05 and mma.sync
// take both operands of one product in the same type, so V must be fp16 too.
// Converting it once per token, when the token enters the cache, replaces a
// conversion of every gathered tile in every CTA that reads it.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"

namespace hga {

// v, out: [Hkv][t_cap][D]; tokens [t_begin, t_end) of every head, 8 values
// (16 bytes) per thread and step.  out may equal v (each thread reads its 16
// bytes before writing them).
template <int D>
__global__ void __launch_bounds__(256) convert_v_kernel(const __nv_bfloat16* v, __half* out,
                                                        int64_t t_cap, int64_t t_begin,
                                                        int64_t t_end, int Hkv) {
  griddep_wait();
  const int64_t per_head = (t_end - t_begin) * (D / 8);
  const int64_t n = per_head * Hkv;
  bool overflow = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = i / per_head, c = i - h * per_head;
    const int64_t off = (h * t_cap + t_begin) * D + c * 8;
    uint4 raw = *reinterpret_cast<const uint4*>(v + off);
    uint32_t* w = reinterpret_cast<uint32_t*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      overflow |= (fabsf(f.x) > 65504.f) | (fabsf(f.y) > 65504.f);
      const __half2 hv = __floats2half2_rn(f.x, f.y);
      w[j] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    *reinterpret_cast<uint4*>(out + off) = raw;
  }
  griddep_launch();
  if (overflow) report(HGA_ERR_DEVICE_CHECK);
}

}  // namespace hga
