// Host-memory tier (tiered KV storage).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.2 (segment-wise
// backward and tiered KV storage): only the active segment stays in VRAM;
// older K/V live in RAM and HGA loads a bounded set of exact historical
// tokens per query block; section 2.1: chunk summaries stay in VRAM, group
// summaries sit in a larger VRAM cache with misses fetched from RAM; section
// 4.5 reports the cache hit rate.
//
// Layout of the tier (all history = tokens < t_hist):
//   * k_host, v_host, gsum_host: pinned host memory, read by the kernels in
//     place over PCIe ([Hkv][t_cap][d] and [Hkv][t_cap/group][d]);
//   * a direct-mapped HBM cache of group summaries: slot = group % cap per KV
//     head, with a tag (the group it holds, -1 empty) and a claim (the largest
//     group that missed on that slot during the current step, -1 none);
//   * device mirrors of K/V and of the group summaries, in the same layout as
//     the all-HBM path, so routing and attention run unchanged on them.
// Per step: fetch_group_summaries (cache hit -> copy from HBM, miss -> copy
// from host and claim the slot) -> group routing -> gather_history (routed,
// sink and local-window history groups, deduplicated per (KV head, group) with
// a generation stamp, on a side stream) -> attention -> install (each claimed
// slot takes its claim).  Installing after the step keeps every lookup of a
// step on the same cache state, so results do not depend on CTA order.
#pragma once
#include "common.cuh"

namespace hga {

struct TierArgs {
  int64_t q_start, n_q, t_cap, t_hist;
  int n_blocks, Hkv, chunk, group, qblock, sink, local;
  int64_t n_groups_cap;     // t_cap / group
  int64_t in_cap;           // chunk_idx slots
  int64_t cap_g;            // group_idx slots
  int64_t cache_cap;        // cache slots per KV head
};

// Copies one 8-token group (or one summary row) of `bytes` with a warp.
__device__ __forceinline__ void warp_copy(const char* __restrict__ src, char* __restrict__ dst,
                                          int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16)
    *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(src + o);
}

// Group summaries of every kept history chunk of (block, KV head): from the
// cache on a hit, from host memory on a miss (and the slot is claimed).
template <int D, typename T>
__global__ void __launch_bounds__(256) fetch_group_summaries_kernel(
    TierArgs a, const int32_t* __restrict__ chunk_idx, const int32_t* __restrict__ chunk_cnt,
    const T* __restrict__ gsum_host, const T* __restrict__ cache_data,
    const int32_t* __restrict__ tags, int32_t* __restrict__ claims, T* __restrict__ gsum_dev,
    unsigned long long* __restrict__ stats) {
  griddep_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int cnt = chunk_cnt[(int64_t)h * a.n_blocks + b];
  if (cnt < 0 || cnt > a.in_cap) {
    if (threadIdx.x == 0) report(HGA_ERR_DEVICE_CHECK);
    return;
  }
  const int per = a.chunk / a.group;
  const int32_t* kept = chunk_idx + ((int64_t)h * a.n_blocks + b) * a.in_cap;
  unsigned long long hits = 0, misses = 0;
  for (int w = warp; w < cnt * per; w += 8) {
    const int c = kept[w / per];
    const int64_t j = (int64_t)c * per + w % per;
    if (c < 0 || (j + 1) * a.group > a.t_hist) continue;     // resident (or invalid: routing reports)
    const int64_t slot = j % a.cache_cap;
    const bool hit = tags[(int64_t)h * a.cache_cap + slot] == j;
    const T* src = hit ? cache_data + ((int64_t)h * a.cache_cap + slot) * D
                       : gsum_host + ((int64_t)h * a.n_groups_cap + j) * D;
    warp_copy(reinterpret_cast<const char*>(src),
              reinterpret_cast<char*>(gsum_dev + ((int64_t)h * a.n_groups_cap + j) * D),
              D * (int)sizeof(T), lane);
    if (lane == 0) {
      if (hit) ++hits;
      else {
        ++misses;
        atomicMax(&claims[(int64_t)h * a.cache_cap + slot], (int)j);
      }
    }
  }
  griddep_launch();
  if (lane == 0 && stats && (hits | misses)) {
    atomicAdd(&stats[0], hits);
    atomicAdd(&stats[1], misses);
  }
}

// History K/V groups needed by (block, KV head): sink, routed and local
// window groups that lie below t_hist.  The first CTA to stamp a group with
// this step's generation copies it; the others skip it.
template <int D, typename T>
__global__ void __launch_bounds__(256) gather_history_kernel(
    TierArgs a, const int32_t* __restrict__ group_idx, const int32_t* __restrict__ group_cnt,
    const T* __restrict__ k_host, const T* __restrict__ v_host, T* __restrict__ k_dev,
    T* __restrict__ v_dev, uint32_t* __restrict__ gen, uint32_t step,
    unsigned long long* __restrict__ bytes) {
  griddep_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int g = a.group;
  const int64_t sink_end = min((int64_t)a.sink, b0);
  const int n_s = (int)(sink_end / g);
  int n_r = group_cnt[(int64_t)h * a.n_blocks + b];
  if (n_r < 0 || n_r > a.cap_g) n_r = 0;
  const int32_t* routed = group_idx + ((int64_t)h * a.n_blocks + b) * a.cap_g;
  const int64_t loc_lo = max(sink_end, b0 - a.local);
  const int n_l = (int)((b0 - loc_lo) / g);
  unsigned long long copied = 0;
  for (int i = warp; i < n_s + n_r + n_l; i += 8) {
    int64_t j;
    if (i < n_s) j = i;
    else if (i < n_s + n_r) j = routed[i - n_s];
    else j = loc_lo / g + (i - n_s - n_r);
    if (j < 0 || (j + 1) * g > a.t_hist) continue;            // resident, or invalid
    uint32_t prev = 0;
    if (lane == 0) prev = atomicExch(&gen[(int64_t)h * a.n_groups_cap + j], step);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == step) continue;                               // already fetched this step
    const int64_t off = ((int64_t)h * a.t_cap + j * g) * D;
    warp_copy(reinterpret_cast<const char*>(k_host + off), reinterpret_cast<char*>(k_dev + off),
              g * D * (int)sizeof(T), lane);
    warp_copy(reinterpret_cast<const char*>(v_host + off), reinterpret_cast<char*>(v_dev + off),
              g * D * (int)sizeof(T), lane);
    copied += 2ull * g * D * sizeof(T);
  }
  griddep_launch();
  if (lane == 0 && bytes && copied) atomicAdd(bytes, copied);
}

// gather_history_kernel with a file-backed store's page cache as the source
// (section 2.2: RAM as a bounded page cache over the disk store).  The host
// made every page the step needs resident (hga_store_prepare); page_table
// maps (KV head, page) to its cache slot, whose image is the page's K half
// then its V half, [page_tokens][D] each.  A group whose page is absent sets
// the device check and is skipped.
struct StoreArgs {
  const char* cache;             // host page cache (pinned, read over PCIe)
  const int32_t* page_table;     // [Hkv][n_pages]
  int64_t n_pages, page_tokens, cache_pages, half_bytes;
};

template <int D, typename T>
__global__ void __launch_bounds__(256) gather_store_kernel(
    TierArgs a, StoreArgs sa, const int32_t* __restrict__ group_idx,
    const int32_t* __restrict__ group_cnt, T* __restrict__ k_dev, T* __restrict__ v_dev,
    uint32_t* __restrict__ gen, uint32_t step, unsigned long long* __restrict__ bytes) {
  griddep_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int g = a.group;
  const int64_t sink_end = min((int64_t)a.sink, b0);
  const int n_s = (int)(sink_end / g);
  int n_r = group_cnt[(int64_t)h * a.n_blocks + b];
  if (n_r < 0 || n_r > a.cap_g) n_r = 0;
  const int32_t* routed = group_idx + ((int64_t)h * a.n_blocks + b) * a.cap_g;
  const int64_t loc_lo = max(sink_end, b0 - a.local);
  const int n_l = (int)((b0 - loc_lo) / g);
  unsigned long long copied = 0;
  for (int i = warp; i < n_s + n_r + n_l; i += 8) {
    int64_t j;
    if (i < n_s) j = i;
    else if (i < n_s + n_r) j = routed[i - n_s];
    else j = loc_lo / g + (i - n_s - n_r);
    if (j < 0 || (j + 1) * g > a.t_hist) continue;            // resident, or invalid
    const int64_t t = j * g;
    const int64_t pg = t / sa.page_tokens;
    const int32_t slot = pg < sa.n_pages ? sa.page_table[(int64_t)h * sa.n_pages + pg] : -1;
    if (slot < 0 || slot >= sa.cache_pages) {
      if (lane == 0) report(HGA_ERR_DEVICE_CHECK);
      continue;
    }
    uint32_t prev = 0;
    if (lane == 0) prev = atomicExch(&gen[(int64_t)h * a.n_groups_cap + j], step);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == step) continue;                               // already fetched this step
    const char* page = sa.cache + (int64_t)slot * 2 * sa.half_bytes +
                       (t - pg * sa.page_tokens) * D * (int64_t)sizeof(T);
    const int64_t off = ((int64_t)h * a.t_cap + t) * D;
    warp_copy(page, reinterpret_cast<char*>(k_dev + off), g * D * (int)sizeof(T), lane);
    warp_copy(page + sa.half_bytes, reinterpret_cast<char*>(v_dev + off),
              g * D * (int)sizeof(T), lane);
    copied += 2ull * g * D * sizeof(T);
  }
  griddep_launch();
  if (lane == 0 && bytes && copied) atomicAdd(bytes, copied);
}

// Each claimed slot takes its claim (the largest group that missed on it).
template <int D, typename T>
__global__ void __launch_bounds__(256) install_group_cache_kernel(
    TierArgs a, const T* __restrict__ gsum_host, T* __restrict__ cache_data,
    int32_t* __restrict__ tags, int32_t* __restrict__ claims) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t slot_all = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (slot_all >= (int64_t)a.Hkv * a.cache_cap) return;
  const int64_t h = slot_all / a.cache_cap;
  const int32_t j = claims[slot_all];
  if (j < 0 || j >= a.n_groups_cap) return;
  warp_copy(reinterpret_cast<const char*>(gsum_host + (h * a.n_groups_cap + j) * D),
            reinterpret_cast<char*>(cache_data + slot_all * D), D * (int)sizeof(T), lane);
  __syncwarp();
  if (lane == 0) {
    tags[slot_all] = j;
    claims[slot_all] = -1;
  }
}

}  // namespace hga
