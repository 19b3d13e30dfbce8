// Step 1: chunk and group summaries (mean of post-RoPE keys).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: HGA keeps a
// summary of every closed 64-token chunk (resident) and of every 8-token
// group, built from the model's projected keys.  The summary is the mean key.
//
// One CTA per (chunk, KV head), one warp per 8-token group.  Every lane issues
// all of its 16-byte loads before the first add (a d=128 bf16 row is 16 lanes
// x 16 B, so a warp load covers two rows = 512 contiguous bytes and a group is
// 4 loads per lane), so a CTA costs about one HBM round trip.  Sums are float64:
// exact for bf16 inputs (64 values of 8 significant bits fit the 53-bit
// significand), so the order of the adds does not matter.  Each mean is
// rounded once to the storage dtype.  The chunk sum is the sum of its group
// sums, staged in shared memory.  HBM-bound: bytes = keys read + summaries
// written.
#pragma once
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"

namespace hga {

constexpr int kSumGroup = 8;        // tokens per group (validated on the host)
constexpr int kSumGroupsPerChunk = 8;

// With vout (bf16 keys only), the CTA also stores its chunk's V tokens below
// t_end as fp16 into vout (same [Hkv][t_cap][D] layout): the commit of a
// segment in one launch.  Its loads are issued before the key loads so the
// two round trips overlap.  A magnitude above 65504 becomes inf and raises
// the device check.
template <typename T, int D>
__global__ void __launch_bounds__(32 * kSumGroupsPerChunk) summaries_kernel(
    const T* __restrict__ k, int64_t t_cap, int64_t c_first, int64_t t_end,
    T* __restrict__ csum, T* __restrict__ gsum, const T* __restrict__ v,
    __half* __restrict__ vout) {
  constexpr int kVec = Elt<T>::kVec;
  constexpr int kLanesPerRow = D / kVec;          // lanes covering one token row
  constexpr int kRowsPerIter = 32 / kLanesPerRow; // rows per warp load
  constexpr int kIters = kSumGroup / kRowsPerIter;
  constexpr int kChunk = kSumGroup * kSumGroupsPerChunk;
  __shared__ double s_gsum[kSumGroupsPerChunk][D];

  griddep_wait();
  griddep_launch();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int64_t c = c_first + blockIdx.x;
  const int64_t tg = c * kChunk + (int64_t)warp * kSumGroup;
  const bool group_closed = tg + kSumGroup <= t_end;
  const bool chunk_closed = (c + 1) * kChunk <= t_end;
  const int col = (lane % kLanesPerRow) * kVec;
  const int sub = lane / kLanesPerRow;
  const T* kh = k + (int64_t)h * t_cap * D;

  // V of this chunk: kChunk rows x D/8 16-byte pieces over the CTA's threads
  constexpr int kVPieces = kChunk * D / 8;
  constexpr int kVPer = kVPieces / (32 * kSumGroupsPerChunk);
  static_assert(kVPieces % (32 * kSumGroupsPerChunk) == 0, "V pieces per thread");
  uint4 vr[kVPer];
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (vout) {
#pragma unroll
      for (int x = 0; x < kVPer; ++x) {
        const int piece = threadIdx.x + x * 32 * kSumGroupsPerChunk;
        const int64_t t = c * kChunk + piece / (D / 8);
        if (t < t_end)
          vr[x] = __ldg(reinterpret_cast<const uint4*>(v + ((int64_t)h * t_cap + t) * D +
                                                       (piece % (D / 8)) * 8));
      }
    }
  }

  double acc[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) acc[i] = 0.0;
  if (group_closed) {
    uint4 raw[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it)
      raw[it] = __ldg(reinterpret_cast<const uint4*>(kh + (tg + it * kRowsPerIter + sub) * D + col));
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      double w[kVec];
      Elt<T>::widen(raw[it], w);
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] += w[i];
    }
#pragma unroll
    for (int off = kLanesPerRow; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    if (lane < kLanesPerRow) {
      __align__(16) T out[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        out[i] = Elt<T>::from_f64(acc[i] / kSumGroup);
        s_gsum[warp][col + i] = acc[i];
      }
      *reinterpret_cast<uint4*>(gsum + ((int64_t)h * (t_cap / kSumGroup) + tg / kSumGroup) * D + col) =
          *reinterpret_cast<const uint4*>(out);
    }
  }
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (vout) {
      bool overflow = false;
#pragma unroll
      for (int x = 0; x < kVPer; ++x) {
        const int piece = threadIdx.x + x * 32 * kSumGroupsPerChunk;
        const int64_t t = c * kChunk + piece / (D / 8);
        if (t >= t_end) continue;
        uint32_t* w = reinterpret_cast<uint32_t*>(&vr[x]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
          overflow |= (fabsf(f.x) > 65504.f) | (fabsf(f.y) > 65504.f);
          const __half2 hv = __floats2half2_rn(f.x, f.y);
          w[j] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(vout + ((int64_t)h * t_cap + t) * D + (piece % (D / 8)) * 8) =
            vr[x];
      }
      if (overflow) report(HGA_ERR_DEVICE_CHECK);
    }
  }
  if (!chunk_closed) return;          // uniform across the CTA
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int g = 0; g < kSumGroupsPerChunk; ++g) s += s_gsum[g][i];
    csum[((int64_t)h * (t_cap / kChunk) + c) * D + i] = Elt<T>::from_f64(s / kChunk);
  }
}

}  // namespace hga
