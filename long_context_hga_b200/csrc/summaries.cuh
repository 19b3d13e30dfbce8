// Step 1: chunk and group summaries (mean of post-RoPE keys).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: HGA keeps a
// summary of every closed 64-token chunk (resident) and of every 8-token
// group, built from the model's projected keys.  The summary is the mean key.
//
// One warp per (KV head, chunk).  The warp streams the chunk's rows with
// coalesced 16-byte loads (a d=128 bf16 row is 16 lanes x 16 B, so one load
// instruction covers two rows = 512 contiguous bytes), sums each group in
// float64 (exact for bf16 inputs: 64 values of 8 significant bits fit the
// 53-bit significand), reduces across the lanes holding the same dims, and
// rounds each mean once to the storage dtype.  The chunk sum is the sum of its
// group sums.  HBM-bound: bytes = keys read + summaries written.
#pragma once
#include "common.cuh"

namespace hga {

template <typename T, int D>
__global__ void __launch_bounds__(256) summaries_kernel(
    const T* __restrict__ k, int64_t t_cap, int n_kv_heads, int64_t c_first,
    int64_t n_chunks, int64_t t_end, int chunk, int group,
    T* __restrict__ csum, T* __restrict__ gsum) {
  constexpr int kVec = Elt<T>::kVec;
  constexpr int kLanesPerRow = D / kVec;          // lanes covering one token row
  constexpr int kRowsPerIter = 32 / kLanesPerRow; // rows per warp load
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (warp >= (int64_t)n_kv_heads * n_chunks) return;
  const int h = (int)(warp / n_chunks);
  const int64_t c = c_first + warp % n_chunks;
  const int64_t t0 = c * chunk;
  const int col = (lane % kLanesPerRow) * kVec;
  const int sub = lane / kLanesPerRow;
  const T* kh = k + (int64_t)h * t_cap * D;
  const int64_t n_groups_cap = t_cap / group;

  double csum_acc[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) csum_acc[i] = 0.0;
  bool chunk_full = (t0 + chunk) <= t_end;

  for (int gi = 0; gi < chunk / group; ++gi) {
    const int64_t tg = t0 + (int64_t)gi * group;
    if (tg + group > t_end) break;           // group not closed: no summary
    double acc[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) acc[i] = 0.0;
    for (int it = 0; it < group / kRowsPerIter; ++it) {
      const int64_t t = tg + it * kRowsPerIter + sub;
      uint4 raw = __ldg(reinterpret_cast<const uint4*>(kh + t * D + col));
      double w[kVec];
      Elt<T>::widen(raw, w);
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] += w[i];
    }
#pragma unroll
    for (int off = kLanesPerRow; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    if (lane < kLanesPerRow) {
      const int64_t j = tg / group;
      __align__(16) T out[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) out[i] = Elt<T>::from_f64(acc[i] / group);
      *reinterpret_cast<uint4*>(gsum + ((int64_t)h * n_groups_cap + j) * D + col) =
          *reinterpret_cast<const uint4*>(out);
    }
#pragma unroll
    for (int i = 0; i < kVec; ++i) csum_acc[i] += acc[i];
  }
  if (chunk_full && lane < kLanesPerRow) {
    __align__(16) T out[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) out[i] = Elt<T>::from_f64(csum_acc[i] / chunk);
    *reinterpret_cast<uint4*>(csum + ((int64_t)h * (t_cap / chunk) + c) * D + col) =
        *reinterpret_cast<const uint4*>(out);
  }
}

}  // namespace hga
