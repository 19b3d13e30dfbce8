// Device storage of the allocation-free history gather.
//
// hga_gather_history takes its per-(KV head, group) generation stamps from
// the caller.  Some callers cannot hand over such a buffer: a runtime that
// sizes all device memory once at start-up (so that a long run has a fixed
// footprint and no step can fail on an allocation), or a host program that
// has no CUDA allocator of its own and only passes this library the mirrors
// and index lists it already owns.  For them hga_gather_history_noalloc keeps
// the stamps in the fixed array below, which the CUDA module reserves when it
// loads; nothing is allocated at call time.
#pragma once
#include <cstdint>

namespace hga {

// 2^18 stamps (1 MiB): n_kv_heads * (t_cap / group) must not exceed this,
// e.g. 8 KV heads x 262144 tokens of capacity with 8-token groups.
constexpr int64_t kStaticGenWords = int64_t(1) << 18;

static __device__ __align__(256) uint32_t g_static_gen[kStaticGenWords];

// Zeroes the first n stamps: every call starts from "nothing copied yet".
__global__ void __launch_bounds__(256) clear_stamps_kernel(uint32_t* __restrict__ w, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) w[i] = 0;
}

}  // namespace hga
