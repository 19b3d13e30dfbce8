// libhga: C ABI entry points (declared in include/hga.h).  Host-side argument
// checks, launch sizing and the device status word; the kernels live in the
// included .cuh files.  One translation unit so that the status word is a
// single device symbol without relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <mutex>

#include "hga.h"
#include "kv_store.h"
#include "common.cuh"
#include "summaries.cuh"
#include "route.cuh"
#include "attend.cuh"
#include "attend_tc.cuh"
#include "attend_bwd.cuh"
#include "attend_bwd_tc.cuh"
#include "route_tc.cuh"
#include "tier.cuh"
#include "noalloc.cuh"
#include "convert_v.cuh"

namespace {

std::atomic<int64_t> g_launches{0};
thread_local cudaError_t g_last_cuda = cudaSuccess;

inline hga_status cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return HGA_OK;
  g_last_cuda = e;
  return HGA_ERR_CUDA;
}

inline hga_status after_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cuda_ok(cudaGetLastError());
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream drains; the kernels call
// griddepcontrol.wait before reading anything (see common.cuh).
template <typename... KArgs, typename... Args>
hga_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_ok(e);
  }
  return cuda_ok(cudaGetLastError());
}

// Opt every kernel into all the dynamic shared memory a block may use (227 KB
// minus the kernel's static shared memory), once per device (the attribute
// belongs to the device context).
constexpr size_t kMaxSmemPerBlock = 227 * 1024;

template <auto kernel>
hga_status allow_smem(size_t bytes) {
  static std::atomic<uint64_t> done{0};
  static std::atomic<size_t> dyn_max{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_ok(e);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(done.load(std::memory_order_acquire) & bit)) {
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return cuda_ok(e);
    const size_t avail = kMaxSmemPerBlock - fa.sharedSizeBytes;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)avail)) != cudaSuccess)
      return cuda_ok(e);
    dyn_max.store(avail, std::memory_order_relaxed);
    done.fetch_or(bit, std::memory_order_acq_rel);
  }
  return bytes <= dyn_max.load(std::memory_order_relaxed) ? HGA_OK : HGA_ERR_UNSUPPORTED;
}

hga_status check_params(const hga_params* p) {
  if (!p) return HGA_ERR_INVALID_ARG;
  if (p->n_q_heads <= 0 || p->n_kv_heads <= 0 || p->n_q_heads % p->n_kv_heads) return HGA_ERR_INVALID_ARG;
  if (p->head_dim <= 0 || p->chunk <= 0 || p->group <= 0 || p->qblock <= 0) return HGA_ERR_INVALID_ARG;
  if (p->chunk % p->group) return HGA_ERR_INVALID_ARG;
  if (p->sink < 0 || p->local < 0 || p->sink % p->chunk || p->local % p->chunk) return HGA_ERR_INVALID_ARG;
  if (p->dtype != HGA_BF16 && p->dtype != HGA_FP32) return HGA_ERR_INVALID_ARG;
  if (p->v_f16 != 0 && p->v_f16 != 1) return HGA_ERR_INVALID_ARG;
  if (p->v_f16 && p->dtype != HGA_BF16) return HGA_ERR_INVALID_ARG;
  if (p->q_ready != 0 && p->q_ready != 1) return HGA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return HGA_ERR_UNSUPPORTED;
  if (p->chunk != 64 || p->group != 8 || p->qblock != 64) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

inline int64_t cap_chunks(const hga_params* p, int64_t t_cap) {
  const int64_t n = t_cap / p->chunk;
  return p->top_chunks > 0 ? std::min<int64_t>(p->top_chunks, n) : n;
}
inline int64_t cap_groups(const hga_params* p, int64_t t_cap) {
  const int64_t n = cap_chunks(p, t_cap) * (p->chunk / p->group);
  return p->top_groups > 0 ? std::min<int64_t>(p->top_groups, n) : n;
}

hga_status check_segment(const hga_params* p, int64_t q_start, int64_t n_q, int64_t t_cap) {
  if (q_start < 0 || n_q < 0 || t_cap <= 0) return HGA_ERR_INVALID_ARG;
  if (q_start % p->qblock) return HGA_ERR_INVALID_ARG;
  if (q_start + n_q > t_cap) return HGA_ERR_INVALID_ARG;
  if ((n_q + p->qblock - 1) / p->qblock > 65535) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

// ---------------------------------------------------------------- TMA maps

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  fn.store(f, std::memory_order_release);
  return f;
}

// bf16 tensor map with the 128-byte swizzle; dims/box innermost first,
// strides in bytes for dims 1..rank-1.  Out-of-range elements read as zero.
bool encode_bf16_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
             reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides),
             reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 0 = choose, 1 = portable mma.sync kernels, 2 = tcgen05 kernels (when eligible)
std::atomic<int> g_kernel_variant{0};

// ---------------------------------------------------------------- routing

bool route_tc_eligible(const hga::RouteArgs& a, const void* q, const void* summ) {
  const uintptr_t align = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(summ);
  return (align & 15) == 0 && (a.G == 1 || a.G == 2 || a.G == 4 || a.G == 8) &&
         a.max_cands <= hga::kRtMaxCands && (int64_t)a.Hkv * a.n_summ_cap < (1ll << 31) &&
         a.n_q < (1ll << 31);
}

template <int D>
hga_status launch_route_tc(hga::RouteArgs& a, cudaStream_t st) {
  using L = hga::RtLayout<D>;
  hga_status s = a.q_early ? allow_smem<hga::route_tc_kernel<D, true>>(L::kSmem)
                           : allow_smem<hga::route_tc_kernel<D, false>>(L::kSmem);
  if (s != HGA_OK) return s;
  hga::RtArgs ra{a, std::min(256, 64 * a.G)};
  CUtensorMap tq, ts, ts8;
  const uint64_t qd[3] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.n_q};
  const uint64_t qs[2] = {(uint64_t)D * 2, (uint64_t)a.Hq * D * 2};
  const uint32_t qb[3] = {64, (uint32_t)a.G, (uint32_t)(ra.rs / a.G)};
  const uint64_t sd[2] = {(uint64_t)D, (uint64_t)a.Hkv * a.n_summ_cap};
  const uint64_t ss[1] = {(uint64_t)D * 2};
  const uint32_t sb[2] = {64, (uint32_t)hga::kRtTile};
  const uint32_t sb8[2] = {64, 8};
  if (!encode_bf16_map(&tq, a.q, 3, qd, qs, qb) || !encode_bf16_map(&ts, a.summ, 2, sd, ss, sb) ||
      !encode_bf16_map(&ts8, a.summ, 2, sd, ss, sb8))
    return HGA_ERR_CUDA;
  dim3 grid(a.n_blocks, a.Hkv);
  if (a.q_early)
    return launch_pdl(hga::route_tc_kernel<D, true>, grid, dim3(hga::kRtThreads), L::kSmem, st,
                      tq, ts, ts8, ra);
  return launch_pdl(hga::route_tc_kernel<D, false>, grid, dim3(hga::kRtThreads), L::kSmem, st, tq,
                    ts, ts8, ra);
}

template <int D>
hga_status launch_route_fused_tc(const hga::RouteArgs& ac, const hga::RouteArgs& ag,
                                 cudaStream_t st) {
  using L = hga::RtLayout<D>;
  hga_status s = allow_smem<hga::route_fused_tc_kernel<D>>(L::kSmem);
  if (s != HGA_OK) return s;
  hga::RtFusedArgs fa{ac, ag, std::min(256, 64 * ac.G)};
  CUtensorMap tq, tc_, tg8;
  const uint64_t qd[3] = {(uint64_t)D, (uint64_t)ac.Hq, (uint64_t)ac.n_q};
  const uint64_t qs[2] = {(uint64_t)D * 2, (uint64_t)ac.Hq * D * 2};
  const uint32_t qb[3] = {64, (uint32_t)ac.G, (uint32_t)(fa.rs / ac.G)};
  const uint64_t cd[2] = {(uint64_t)D, (uint64_t)ac.Hkv * ac.n_summ_cap};
  const uint64_t gd[2] = {(uint64_t)D, (uint64_t)ag.Hkv * ag.n_summ_cap};
  const uint64_t ss[1] = {(uint64_t)D * 2};
  const uint32_t cb[2] = {64, (uint32_t)hga::kRtTile};
  const uint32_t gb[2] = {64, 8};
  if (!encode_bf16_map(&tq, ac.q, 3, qd, qs, qb) || !encode_bf16_map(&tc_, ac.summ, 2, cd, ss, cb) ||
      !encode_bf16_map(&tg8, ag.summ, 2, gd, ss, gb))
    return HGA_ERR_CUDA;
  dim3 grid(ac.n_blocks, ac.Hkv);
  return launch_pdl(hga::route_fused_tc_kernel<D>, grid, dim3(hga::kRtThreads), L::kSmem, st, tq,
                    tc_, tg8, fa);
}

constexpr int kMaxRouteCands = 16384;
constexpr int kMaxKeptChunks = 2048;

template <typename T, int D>
hga_status launch_route(hga::RouteArgs& a, cudaStream_t st) {
  const size_t smem = hga::route_smem_bytes<T, D>(a.max_cands);
  hga_status s = allow_smem<hga::route_kernel<T, D>>(smem);
  if (s != HGA_OK) return s;
  dim3 grid(a.n_blocks, a.Hkv);
  return launch_pdl(hga::route_kernel<T, D>, grid, dim3(hga::kRouteThreads), smem, st, a);
}

// Arguments of one routing step; HGA_OK with a.n_q == 0 means nothing to do.
hga_status route_args(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                      const void* summ, int64_t t_cap, const int32_t* in_idx,
                      const int32_t* in_cnt, int32_t* out_idx, int32_t* out_cnt, int group_mode,
                      hga::RouteArgs& a) {
  a = hga::RouteArgs{};
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if ((s = check_segment(p, q_start, n_q, t_cap)) != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!q || !summ || !out_idx || !out_cnt || (group_mode && (!in_idx || !in_cnt)))
    return HGA_ERR_INVALID_ARG;
  a.q = q;
  a.q_start = q_start;
  a.n_q = n_q;
  a.summ = summ;
  a.n_blocks = (int)((n_q + p->qblock - 1) / p->qblock);
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.G = p->n_q_heads / p->n_kv_heads;
  a.chunk = p->chunk;
  a.group = p->group;
  a.qblock = p->qblock;
  a.sink = p->sink;
  a.local = p->local;
  a.group_mode = group_mode;
  a.q_early = p->q_ready;
  a.in_idx = in_idx;
  a.in_cnt = in_cnt;
  a.out_idx = out_idx;
  a.out_cnt = out_cnt;
  const int per = p->chunk / p->group;
  if (!group_mode) {
    a.n_summ_cap = t_cap / p->chunk;
    a.in_cap = 0;
    a.out_cap = cap_chunks(p, t_cap);
    a.top_k = p->top_chunks;
    const int64_t last_b0 = q_start + (int64_t)(a.n_blocks - 1) * p->qblock;
    const int64_t hi = last_b0 - p->local > 0 ? (last_b0 - p->local) / p->chunk : 0;
    const int64_t n = std::max<int64_t>(0, hi - p->sink / p->chunk);
    if (n > kMaxRouteCands) return HGA_ERR_UNSUPPORTED;
    a.max_cands = (int)std::max<int64_t>(n, 1);
  } else {
    a.n_summ_cap = t_cap / p->group;
    a.in_cap = cap_chunks(p, t_cap);
    a.out_cap = cap_groups(p, t_cap);
    a.top_k = p->top_groups;
    if (a.in_cap > kMaxKeptChunks || a.in_cap * per > kMaxRouteCands) return HGA_ERR_UNSUPPORTED;
    a.max_cands = (int)std::max<int64_t>(a.in_cap * per, 1);
  }
  return HGA_OK;
}

hga_status route_common(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                        const void* summ, int64_t t_cap, const int32_t* in_idx,
                        const int32_t* in_cnt, int32_t* out_idx, int32_t* out_cnt, int group_mode,
                        cudaStream_t st) {
  hga::RouteArgs a;
  hga_status s = route_args(p, q, q_start, n_q, summ, t_cap, in_idx, in_cnt, out_idx, out_cnt,
                            group_mode, a);
  if (s != HGA_OK || n_q == 0) return s;
  if (p->dtype == HGA_BF16) {
    if (g_kernel_variant.load(std::memory_order_relaxed) != 1 && route_tc_eligible(a, q, summ))
      return p->head_dim == 128 ? launch_route_tc<128>(a, st) : launch_route_tc<64>(a, st);
    return p->head_dim == 128 ? launch_route<__nv_bfloat16, 128>(a, st)
                              : launch_route<__nv_bfloat16, 64>(a, st);
  }
  return p->head_dim == 128 ? launch_route<float, 128>(a, st) : launch_route<float, 64>(a, st);
}

template <typename T, int D>
hga_status launch_summaries(const void* k, int64_t t_cap, int Hkv, int64_t t_begin, int64_t t_end,
                            int chunk, int group, void* cs, void* gs, cudaStream_t st,
                            const void* v = nullptr, void* v_f16 = nullptr) {
  const int64_t c_first = t_begin / chunk;
  const int64_t c_last = (t_end + chunk - 1) / chunk;   // partial chunk: its closed groups
  const int64_t n_chunks = c_last - c_first;
  if (n_chunks <= 0) return HGA_OK;
  if (n_chunks > 0x7fffffff || Hkv > 65535) return HGA_ERR_UNSUPPORTED;
  (void)chunk;
  (void)group;   // 64 / 8, validated by check_params
  dim3 grid((unsigned)n_chunks, Hkv);
  return launch_pdl(hga::summaries_kernel<T, D>, grid, dim3(32 * hga::kSumGroupsPerChunk), 0, st,
                    reinterpret_cast<const T*>(k), t_cap, c_first, t_end, reinterpret_cast<T*>(cs),
                    reinterpret_cast<T*>(gs), reinterpret_cast<const T*>(v),
                    reinterpret_cast<__half*>(v_f16));
}

// One-shot test hook: the next tensor-core attention launch stops loading
// K/V at this ring index (-1: off).  See hga_debug_stall_next_attend.
std::atomic<int64_t> g_stall_next_attend{-1};

template <int D, bool VF16>
hga_status launch_attend_tc(hga::AttendArgs& a, cudaStream_t st) {
  using L = hga::TcLayout<D>;
  const size_t smem = L::smem_bytes(a.max_list);
  hga_status s = allow_smem<hga::attend_tc_kernel<D, VF16>>(smem);
  if (s != HGA_OK) return s;
  CUtensorMap tq, tk1, tk8, tv1, tv8, to;
  const uint64_t qd[3] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.n_q};
  const uint64_t qs[2] = {(uint64_t)D * 2, (uint64_t)a.Hq * D * 2};
  const uint32_t qb[3] = {64, (uint32_t)a.G, (uint32_t)(hga::kTcRows / a.G)};
  // O has Q's layout and the epilogue stores a Q tile's rows, but never more
  // positions than one query block holds: with G = 1 a 128-row tile spans two
  // blocks, and the second block's rows belong to another CTA.
  const uint32_t ob[3] = {64, (uint32_t)a.G,
                          (uint32_t)std::min(hga::kTcRows / a.G, a.qblock)};
  if (!encode_bf16_map(&tq, a.q, 3, qd, qs, qb) || !encode_bf16_map(&to, a.o, 3, qd, qs, ob))
    return HGA_ERR_CUDA;
  // K/V as (64 dims, 8 rows, D/64 halves, group): one box = whole groups
  // landing as [group][half][8 rows][128 B].  Tiled TMA copies bytes, so the
  // bf16 map serves fp16 V as well.
  const uint64_t gd[4] = {64, 8, (uint64_t)(D / 64), (uint64_t)a.Hkv * a.t_cap / 8};
  const uint64_t gs[3] = {(uint64_t)D * 2, 128, (uint64_t)D * 2 * 8};
  const uint32_t b1[4] = {64, 8, (uint32_t)(D / 64), 1};
  const uint32_t b8[4] = {64, 8, (uint32_t)(D / 64), 8};
  if (!encode_bf16_map(&tk1, a.k, 4, gd, gs, b1) || !encode_bf16_map(&tk8, a.k, 4, gd, gs, b8) ||
      !encode_bf16_map(&tv1, a.v, 4, gd, gs, b1) || !encode_bf16_map(&tv8, a.v, 4, gd, gs, b8))
    return HGA_ERR_CUDA;
  hga::TcArgs ta{};
  ta.a = a;
  ta.rows_per_cta = 2 * hga::kTcRows;
  ta.stall_load = g_stall_next_attend.exchange(-1, std::memory_order_relaxed);
  dim3 grid((a.qblock * a.G + ta.rows_per_cta - 1) / ta.rows_per_cta, a.n_blocks, a.Hkv);
  return launch_pdl(hga::attend_tc_kernel<D, VF16>, grid, dim3(hga::kTcThreads), smem, st, tq, tk1,
                    tk8, tv1, tv8, to, ta);
}

bool tc_eligible(const hga::AttendArgs& a) {
  const uintptr_t align = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                          reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.o);
  return (align & 15) == 0 && a.G <= hga::kTcRows && (hga::kTcRows % a.G) == 0 &&
         a.max_list <= hga::kTcMaxList && (int64_t)a.Hkv * a.t_cap < (1ll << 31) &&
         a.n_q < (1ll << 31) && (a.t_cap % a.group) == 0;
}

template <int D, bool VF16>
hga_status launch_attend_bf16(hga::AttendArgs& a, cudaStream_t st) {
  const int variant = g_kernel_variant.load(std::memory_order_relaxed);
  if (variant != 1 && tc_eligible(a)) return launch_attend_tc<D, VF16>(a, st);
  const size_t smem = hga::attend_mma_smem_bytes<D>(a.max_list);
  hga_status s = allow_smem<hga::attend_mma_kernel<D, VF16>>(smem);
  if (s != HGA_OK) return s;
  dim3 grid((a.qblock * a.G + hga::kAttRows - 1) / hga::kAttRows, a.n_blocks, a.Hkv);
  return launch_pdl(hga::attend_mma_kernel<D, VF16>, grid, dim3(128), smem, st, a);
}

template <int D>
hga_status launch_attend_f32(hga::AttendArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.max_list * 4;
  hga_status s = allow_smem<hga::attend_f32_kernel<D>>(smem);
  if (s != HGA_OK) return s;
  dim3 grid((a.qblock * a.G + hga::kAttF32Rows - 1) / hga::kAttF32Rows, a.n_blocks, a.Hkv);
  return launch_pdl(hga::attend_f32_kernel<D>, grid, dim3(256), smem, st, a);
}

}  // namespace

template <typename T, int D>
hga_status launch_attend_bwd(hga::BwArgs& w, cudaStream_t st) {
  using L = hga::BwLayout<D>;
  const size_t smem = L::smem_bytes(w.a.max_list);
  hga_status s = allow_smem<hga::attend_bwd_kernel<T, D>>(smem);
  if (s != HGA_OK) return s;
  dim3 grid((unsigned)((w.a.qblock * w.a.G + hga::kBwRows - 1) / hga::kBwRows), w.a.n_blocks,
            w.a.Hkv);
  return launch_pdl(hga::attend_bwd_kernel<T, D>, grid, dim3(hga::kBwThreads), smem, st, w);
}

// Tensor-core backward (bf16): D = rowsum(dO o) into d_q's first column,
// then the dK/dV kernel, then the dQ kernel (see attend_bwd_tc.cuh).  Every
// group in the lists must be whole (the context a multiple of the group
// size): a partial group's tokens past the context would be read from the
// cache as they are.
bool bwd_tc_eligible(const hga::AttendArgs& a, const void* o, const void* d_o) {
  const uintptr_t align = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                          reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(o) |
                          reinterpret_cast<uintptr_t>(d_o);
  return (align & 15) == 0 && a.G <= hga::kBtRows && (hga::kBtRows % a.G) == 0 &&
         a.max_list <= hga::kTcMaxList && (int64_t)a.Hkv * a.t_cap < (1ll << 31) &&
         a.n_q < (1ll << 31) && (a.t_cap % a.group) == 0 && ((a.q_start + a.n_q) % a.group) == 0;
}

template <int D>
hga_status launch_attend_bwd_tc(hga::BtArgs& w, cudaStream_t st) {
  using LK = hga::BtKvLayout<D>;
  using LQ = hga::BtQLayout<D>;
  const hga::AttendArgs& a = w.a;
  hga_status s = allow_smem<hga::bwd_dkdv_kernel<D>>(LK::smem_bytes());
  if (s != HGA_OK) return s;
  if ((s = allow_smem<hga::bwd_dq_kernel<D>>(LQ::smem_bytes(a.max_list))) != HGA_OK) return s;
  CUtensorMap tq, tdo, tk1, tk8, tv1, tv8;
  const uint64_t qd[3] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.n_q};
  const uint64_t qs[2] = {(uint64_t)D * 2, (uint64_t)a.Hq * D * 2};
  const uint32_t qb[3] = {64, (uint32_t)a.G, (uint32_t)(hga::kBtRows / a.G)};
  if (!encode_bf16_map(&tq, a.q, 3, qd, qs, qb) || !encode_bf16_map(&tdo, w.d_o, 3, qd, qs, qb))
    return HGA_ERR_CUDA;
  const uint64_t gd[4] = {64, 8, (uint64_t)(D / 64), (uint64_t)a.Hkv * a.t_cap / 8};
  const uint64_t gs[3] = {(uint64_t)D * 2, 128, (uint64_t)D * 2 * 8};
  const uint32_t b1[4] = {64, 8, (uint32_t)(D / 64), 1};
  const uint32_t b8[4] = {64, 8, (uint32_t)(D / 64), 8};
  if (!encode_bf16_map(&tk1, a.k, 4, gd, gs, b1) || !encode_bf16_map(&tk8, a.k, 4, gd, gs, b8) ||
      !encode_bf16_map(&tv1, a.v, 4, gd, gs, b1) || !encode_bf16_map(&tv8, a.v, 4, gd, gs, b8))
    return HGA_ERR_CUDA;
  const int64_t n_rows = a.n_q * a.Hq;
  const unsigned dblocks = (unsigned)std::min<int64_t>((n_rows + 7) / 8, 1 << 20);
  if ((s = launch_pdl(hga::bwd_dsum_kernel<D>, dim3(dblocks), dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(w.o),
                      static_cast<const __nv_bfloat16*>(w.d_o), w.d_q, n_rows)) != HGA_OK)
    return s;
  const int n_kv_tiles = (a.max_list + hga::kBtGroupsPerTile - 1) / hga::kBtGroupsPerTile;
  dim3 gk((unsigned)n_kv_tiles, a.n_blocks, a.Hkv);
  if ((s = launch_pdl(hga::bwd_dkdv_kernel<D>, gk, dim3(hga::kBtThreads), LK::smem_bytes(), st, tq,
                      tdo, tk1, tk8, tv1, tv8, w)) != HGA_OK)
    return s;
  dim3 gq((unsigned)((a.qblock * a.G + hga::kBtRows - 1) / hga::kBtRows), a.n_blocks, a.Hkv);
  return launch_pdl(hga::bwd_dq_kernel<D>, gq, dim3(hga::kBtThreads), LQ::smem_bytes(a.max_list),
                    st, tq, tdo, tk1, tk8, tv1, tv8, w);
}

// hga_attend with rows of positions before pos_lo allowed to be skipped (the
// tensor-core kernel skips them; the others compute every row).
hga_status attend_impl(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                       const void* k, const void* v, int64_t t_cap, const int32_t* group_idx,
                       const int32_t* group_cnt, void* o, float* lse, int64_t pos_lo,
                       cudaStream_t st) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if ((s = check_segment(p, q_start, n_q, t_cap)) != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!q || !k || !v || !group_idx || !group_cnt || !o) return HGA_ERR_INVALID_ARG;
  hga::AttendArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.q_start = q_start;
  a.n_q = n_q;
  a.t_cap = t_cap;
  a.group_idx = group_idx;
  a.group_cnt = group_cnt;
  a.cap_g = cap_groups(p, t_cap);
  a.o = o;
  a.lse = lse;
  a.n_blocks = (int)((n_q + p->qblock - 1) / p->qblock);
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.G = p->n_q_heads / p->n_kv_heads;
  a.group = p->group;
  a.qblock = p->qblock;
  a.sink = p->sink;
  a.local = p->local;
  a.q_early = p->q_ready;
  const int64_t max_list = p->sink / p->group + a.cap_g + p->local / p->group +
                           (p->qblock + p->group - 1) / p->group;
  if (max_list > 16384) return HGA_ERR_UNSUPPORTED;
  a.max_list = (int)max_list;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)p->head_dim));
  a.pos_lo = pos_lo;
  if (p->dtype == HGA_BF16 && p->v_f16)
    return p->head_dim == 128 ? launch_attend_bf16<128, true>(a, st)
                              : launch_attend_bf16<64, true>(a, st);
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? launch_attend_bf16<128, false>(a, st)
                              : launch_attend_bf16<64, false>(a, st);
  return p->head_dim == 128 ? launch_attend_f32<128>(a, st) : launch_attend_f32<64>(a, st);
}

extern "C" {

hga_status hga_validate_params(const hga_params* p) { return check_params(p); }

int64_t hga_index_capacity(const hga_params* p, int64_t t_cap, int32_t which) {
  if (check_params(p) != HGA_OK || t_cap < 0) return -1;
  if (which == 0) return cap_chunks(p, t_cap);
  if (which == 1) return cap_groups(p, t_cap);
  return -1;
}

hga_status hga_build_summaries(const hga_params* p, const void* k, int64_t t_cap,
                               int64_t t_begin, int64_t t_end, void* chunk_sum,
                               void* group_sum, hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (t_cap <= 0 || t_begin < 0 || t_begin > t_end || t_end > t_cap) return HGA_ERR_INVALID_ARG;
  if (t_begin % p->chunk) return HGA_ERR_INVALID_ARG;
  if (t_begin == t_end) return HGA_OK;
  if (!k || !chunk_sum || !group_sum) return HGA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = p->n_kv_heads;
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128
               ? launch_summaries<__nv_bfloat16, 128>(k, t_cap, Hkv, t_begin, t_end, p->chunk,
                                                      p->group, chunk_sum, group_sum, st)
               : launch_summaries<__nv_bfloat16, 64>(k, t_cap, Hkv, t_begin, t_end, p->chunk,
                                                     p->group, chunk_sum, group_sum, st);
  return p->head_dim == 128
             ? launch_summaries<float, 128>(k, t_cap, Hkv, t_begin, t_end, p->chunk, p->group,
                                            chunk_sum, group_sum, st)
             : launch_summaries<float, 64>(k, t_cap, Hkv, t_begin, t_end, p->chunk, p->group,
                                           chunk_sum, group_sum, st);
}

hga_status hga_commit(const hga_params* p, const void* k, const void* v, int64_t t_cap,
                      int64_t t_begin, int64_t t_end, void* chunk_sum, void* group_sum,
                      void* v_f16, hga_stream_t stream) {
  if (!v_f16) return hga_build_summaries(p, k, t_cap, t_begin, t_end, chunk_sum, group_sum, stream);
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (p->dtype != HGA_BF16) return HGA_ERR_INVALID_ARG;
  if (t_cap <= 0 || t_begin < 0 || t_begin > t_end || t_end > t_cap) return HGA_ERR_INVALID_ARG;
  if (t_begin % p->chunk) return HGA_ERR_INVALID_ARG;
  if (!v || ((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(v_f16)) & 15))
    return HGA_ERR_INVALID_ARG;
  const char* vb = static_cast<const char*>(v);
  const char* ob = static_cast<const char*>(v_f16);
  const int64_t bytes = (int64_t)p->n_kv_heads * t_cap * p->head_dim * 2;
  if (vb != ob && vb < ob + bytes && ob < vb + bytes) return HGA_ERR_INVALID_ARG;
  if (t_begin == t_end) return HGA_OK;
  if (!k || !chunk_sum || !group_sum) return HGA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = p->n_kv_heads;
  return p->head_dim == 128
             ? launch_summaries<__nv_bfloat16, 128>(k, t_cap, Hkv, t_begin, t_end, p->chunk,
                                                    p->group, chunk_sum, group_sum, st, v, v_f16)
             : launch_summaries<__nv_bfloat16, 64>(k, t_cap, Hkv, t_begin, t_end, p->chunk,
                                                   p->group, chunk_sum, group_sum, st, v, v_f16);
}

hga_status hga_route_chunks(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                            const void* chunk_sum, int64_t t_cap, int32_t* chunk_idx,
                            int32_t* chunk_cnt, hga_stream_t stream) {
  return route_common(p, q, q_start, n_q, chunk_sum, t_cap, nullptr, nullptr, chunk_idx,
                      chunk_cnt, 0, reinterpret_cast<cudaStream_t>(stream));
}

hga_status hga_route_groups(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                            const void* group_sum, int64_t t_cap, const int32_t* chunk_idx,
                            const int32_t* chunk_cnt, int32_t* group_idx, int32_t* group_cnt,
                            hga_stream_t stream) {
  return route_common(p, q, q_start, n_q, group_sum, t_cap, chunk_idx, chunk_cnt, group_idx,
                      group_cnt, 1, reinterpret_cast<cudaStream_t>(stream));
}

hga_status hga_attend(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                      const void* k, const void* v, int64_t t_cap, const int32_t* group_idx,
                      const int32_t* group_cnt, void* o, float* lse, hga_stream_t stream) {
  return attend_impl(p, q, q_start, n_q, k, v, t_cap, group_idx, group_cnt, o, lse, q_start,
                     reinterpret_cast<cudaStream_t>(stream));
}

hga_status hga_attend_backward(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                               const void* k, const void* v, int64_t t_cap,
                               const int32_t* group_idx, const int32_t* group_cnt, const void* o,
                               const float* lse, const void* d_o, float* d_q, float* d_k,
                               float* d_v, hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (p->v_f16) return HGA_ERR_INVALID_ARG;
  if ((s = check_segment(p, q_start, n_q, t_cap)) != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!q || !k || !v || !group_idx || !group_cnt || !o || !lse || !d_o || !d_q || !d_k || !d_v)
    return HGA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_k) |
       reinterpret_cast<uintptr_t>(d_v)) & 15)
    return HGA_ERR_INVALID_ARG;
  hga::BwArgs w{};
  hga::AttendArgs& a = w.a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q_start = q_start;
  a.n_q = n_q;
  a.t_cap = t_cap;
  a.group_idx = group_idx;
  a.group_cnt = group_cnt;
  a.cap_g = cap_groups(p, t_cap);
  a.n_blocks = (int)((n_q + p->qblock - 1) / p->qblock);
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.G = p->n_q_heads / p->n_kv_heads;
  a.group = p->group;
  a.qblock = p->qblock;
  a.sink = p->sink;
  a.local = p->local;
  const int64_t max_list = p->sink / p->group + a.cap_g + p->local / p->group +
                           (p->qblock + p->group - 1) / p->group;
  if (max_list > 16384) return HGA_ERR_UNSUPPORTED;
  a.max_list = (int)max_list;
  w.o = o;
  w.d_o = d_o;
  w.lse = lse;
  w.d_q = d_q;
  w.d_k = d_k;
  w.d_v = d_v;
  w.scale = (float)(1.0 / sqrt((double)p->head_dim));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // dK and dV are sums over the query rows that attend each token: start
  // from zero on every head's tokens [0, T)
  const int64_t T = q_start + n_q;
  const size_t row_bytes = (size_t)T * p->head_dim * 4;
  const size_t pitch = (size_t)t_cap * p->head_dim * 4;
  cudaError_t e = cudaMemset2DAsync(d_k, pitch, 0, row_bytes, p->n_kv_heads, st);
  if (e == cudaSuccess) e = cudaMemset2DAsync(d_v, pitch, 0, row_bytes, p->n_kv_heads, st);
  if (e != cudaSuccess) return cuda_ok(e);
  if (p->dtype == HGA_BF16 && g_kernel_variant.load(std::memory_order_relaxed) != 1 &&
      bwd_tc_eligible(a, o, d_o)) {
    hga::BtArgs bt{};
    bt.a = a;
    bt.o = o;
    bt.d_o = d_o;
    bt.lse = lse;
    bt.d_q = d_q;
    bt.d_k = d_k;
    bt.d_v = d_v;
    bt.scale = w.scale;
    bt.scale_log2 = (float)(1.4426950408889634 / sqrt((double)p->head_dim));
    return p->head_dim == 128 ? launch_attend_bwd_tc<128>(bt, st)
                              : launch_attend_bwd_tc<64>(bt, st);
  }
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? launch_attend_bwd<__nv_bfloat16, 128>(w, st)
                              : launch_attend_bwd<__nv_bfloat16, 64>(w, st);
  return p->head_dim == 128 ? launch_attend_bwd<float, 128>(w, st)
                            : launch_attend_bwd<float, 64>(w, st);
}

hga_status hga_route(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                     const void* chunk_sum, const void* group_sum, int64_t t_cap,
                     int32_t* chunk_idx, int32_t* chunk_cnt, int32_t* group_idx,
                     int32_t* group_cnt, hga_stream_t stream) {
  hga::RouteArgs ac, ag;
  hga_status s = route_args(p, q, q_start, n_q, chunk_sum, t_cap, nullptr, nullptr, chunk_idx,
                            chunk_cnt, 0, ac);
  if (s != HGA_OK) return s;
  if ((s = route_args(p, q, q_start, n_q, group_sum, t_cap, chunk_idx, chunk_cnt, group_idx,
                      group_cnt, 1, ag)) != HGA_OK)
    return s;
  if (n_q == 0) return HGA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p->dtype == HGA_BF16 && g_kernel_variant.load(std::memory_order_relaxed) != 1 &&
      route_tc_eligible(ac, q, chunk_sum) && route_tc_eligible(ag, q, group_sum) &&
      ac.out_cap <= 2048)
    return p->head_dim == 128 ? launch_route_fused_tc<128>(ac, ag, st)
                              : launch_route_fused_tc<64>(ac, ag, st);
  s = route_common(p, q, q_start, n_q, chunk_sum, t_cap, nullptr, nullptr, chunk_idx, chunk_cnt,
                   0, st);
  if (s != HGA_OK) return s;
  return route_common(p, q, q_start, n_q, group_sum, t_cap, chunk_idx, chunk_cnt, group_idx,
                      group_cnt, 1, st);
}

hga_status hga_forward(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                       const void* k, const void* v, int64_t t_cap, void* chunk_sum,
                       void* group_sum, int32_t* chunk_idx, int32_t* chunk_cnt,
                       int32_t* group_idx, int32_t* group_cnt, void* o, float* lse,
                       hga_stream_t stream) {
  hga_status s = hga_build_summaries(p, k, t_cap, q_start, q_start + n_q, chunk_sum, group_sum,
                                     stream);
  if (s != HGA_OK) return s;
  s = hga_route_chunks(p, q, q_start, n_q, chunk_sum, t_cap, chunk_idx, chunk_cnt, stream);
  if (s != HGA_OK) return s;
  hga_params pq = *p;     // these follow the library's own routing kernels
  pq.q_ready = 1;
  s = hga_route_groups(&pq, q, q_start, n_q, group_sum, t_cap, chunk_idx, chunk_cnt, group_idx,
                       group_cnt, stream);
  if (s != HGA_OK) return s;
  return hga_attend(&pq, q, q_start, n_q, k, v, t_cap, group_idx, group_cnt, o, lse, stream);
}

hga_status hga_forward_causal(const hga_params* p, const void* q_ext, int64_t q_start,
                              int64_t n_q, const void* k, const void* v, int64_t t_cap,
                              void* chunk_sum, void* group_sum, int32_t* chunk_idx,
                              int32_t* chunk_cnt, int32_t* group_idx, int32_t* group_cnt, void* o,
                              float* lse, hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if ((s = check_segment(p, q_start, n_q, t_cap)) != HGA_OK) return s;
  if (n_q > 0 && !q_ext) return HGA_ERR_INVALID_ARG;
  // routing reads rows [b*qblock, ..) of q_ext = the block before block b;
  // attention reads the segment's own queries, qblock rows further on
  const size_t elem = p->dtype == HGA_BF16 ? 2 : 4;
  const void* q = q_ext ? static_cast<const char*>(q_ext) +
                              (size_t)p->qblock * p->n_q_heads * p->head_dim * elem
                        : nullptr;
  if ((s = hga_build_summaries(p, k, t_cap, q_start, q_start + n_q, chunk_sum, group_sum,
                               stream)) != HGA_OK)
    return s;
  if ((s = hga_route_chunks(p, q_ext, q_start, n_q, chunk_sum, t_cap, chunk_idx, chunk_cnt,
                            stream)) != HGA_OK)
    return s;
  hga_params pq = *p;     // these follow the library's own routing kernels
  pq.q_ready = 1;
  if ((s = hga_route_groups(&pq, q_ext, q_start, n_q, group_sum, t_cap, chunk_idx, chunk_cnt,
                            group_idx, group_cnt, stream)) != HGA_OK)
    return s;
  return hga_attend(&pq, q, q_start, n_q, k, v, t_cap, group_idx, group_cnt, o, lse, stream);
}

hga_status hga_decode_step(const hga_params* p, const void* q_block, int64_t pos, const void* k,
                           const void* v, int64_t t_cap, void* chunk_sum, void* group_sum,
                           int32_t* chunk_idx, int32_t* chunk_cnt, int32_t* group_idx,
                           int32_t* group_cnt, void* v_f16, void* o, float* lse,
                           hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (p->v_f16) return HGA_ERR_INVALID_ARG;       // v is in dtype; v_f16 names the fp16 copy
  if (pos < 0 || pos >= t_cap) return HGA_ERR_INVALID_ARG;
  if (v_f16 && v_f16 == v) return HGA_ERR_INVALID_ARG;
  const int64_t b0 = pos - pos % p->qblock;
  const int64_t n = pos - b0 + 1;
  if ((s = hga_commit(p, k, v, t_cap, b0, pos + 1, chunk_sum, group_sum, v_f16, stream)) != HGA_OK)
    return s;
  if ((s = hga_route_chunks(p, q_block, b0, n, chunk_sum, t_cap, chunk_idx, chunk_cnt, stream)) !=
      HGA_OK)
    return s;
  hga_params pq = *p;     // these follow the library's own routing kernels
  pq.q_ready = 1;
  if ((s = hga_route_groups(&pq, q_block, b0, n, group_sum, t_cap, chunk_idx, chunk_cnt, group_idx,
                            group_cnt, stream)) != HGA_OK)
    return s;
  hga_params pa = pq;
  pa.v_f16 = v_f16 ? 1 : 0;
  // only the token's rows: the other rows of the block are not needed again
  return attend_impl(&pa, q_block, b0, n, k, v_f16 ? v_f16 : v, t_cap, group_idx, group_cnt, o,
                     lse, pos, reinterpret_cast<cudaStream_t>(stream));
}

hga_status hga_check(hga_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_ok(e);
  int st = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&st, hga::g_status, sizeof(int))) != cudaSuccess) return cuda_ok(e);
  if (st != 0 && (e = cudaMemcpyToSymbol(hga::g_status, &zero, sizeof(int))) != cudaSuccess)
    return cuda_ok(e);
  return (hga_status)st;
}

const char* hga_status_string(hga_status s) {
  switch (s) {
    case HGA_OK: return "HGA_OK";
    case HGA_ERR_INVALID_ARG: return "HGA_ERR_INVALID_ARG";
    case HGA_ERR_UNSUPPORTED: return "HGA_ERR_UNSUPPORTED";
    case HGA_ERR_CUDA: return "HGA_ERR_CUDA";
    case HGA_ERR_DEVICE_CHECK: return "HGA_ERR_DEVICE_CHECK";
    case HGA_ERR_TIMEOUT: return "HGA_ERR_TIMEOUT";
    case HGA_ERR_IO: return "HGA_ERR_IO";
    case HGA_ERR_CAPACITY: return "HGA_ERR_CAPACITY";
  }
  return "HGA_ERR_UNKNOWN";
}

int64_t hga_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }


// ---------------------------------------------------------------- host tier

static hga_status tier_args(const hga_params* p, int64_t q_start, int64_t n_q, int64_t t_cap,
                            int64_t t_hist, hga::TierArgs* a) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if ((s = check_segment(p, q_start, n_q, t_cap)) != HGA_OK) return s;
  if (t_hist < 0 || t_hist > q_start || t_hist % p->group) return HGA_ERR_INVALID_ARG;
  *a = hga::TierArgs{};
  a->q_start = q_start;
  a->n_q = n_q;
  a->t_cap = t_cap;
  a->t_hist = t_hist;
  a->n_blocks = (int)((n_q + p->qblock - 1) / p->qblock);
  a->Hkv = p->n_kv_heads;
  a->chunk = p->chunk;
  a->group = p->group;
  a->qblock = p->qblock;
  a->sink = p->sink;
  a->local = p->local;
  a->n_groups_cap = t_cap / p->group;
  a->in_cap = cap_chunks(p, t_cap);
  a->cap_g = cap_groups(p, t_cap);
  return HGA_OK;
}

hga_status hga_fetch_group_summaries(const hga_params* p, int64_t q_start, int64_t n_q,
                                     int64_t t_cap, int64_t t_hist, const int32_t* chunk_idx,
                                     const int32_t* chunk_cnt, const void* group_sum_host,
                                     const hga_group_cache* cache, void* group_sum_dev,
                                     hga_stream_t stream) {
  hga::TierArgs a;
  hga_status s = tier_args(p, q_start, n_q, t_cap, t_hist, &a);
  if (s != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!chunk_idx || !chunk_cnt || !group_sum_host || !cache || !group_sum_dev || !cache->data ||
      !cache->tags || !cache->claims || cache->cap <= 0 || cache->cap > 0x7fffffff)
    return HGA_ERR_INVALID_ARG;
  a.cache_cap = cache->cap;
  dim3 grid(a.n_blocks, a.Hkv);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto go = [&](auto tag, auto dim) {
    using T = decltype(tag);
    constexpr int D = decltype(dim)::value;
    return launch_pdl(hga::fetch_group_summaries_kernel<D, T>, grid, dim3(256), 0, st, a,
                      chunk_idx, chunk_cnt, reinterpret_cast<const T*>(group_sum_host),
                      reinterpret_cast<const T*>(cache->data), (const int32_t*)cache->tags,
                      cache->claims, reinterpret_cast<T*>(group_sum_dev), cache->stats);
  };
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? go(__nv_bfloat16{}, std::integral_constant<int, 128>{})
                              : go(__nv_bfloat16{}, std::integral_constant<int, 64>{});
  return p->head_dim == 128 ? go(float{}, std::integral_constant<int, 128>{})
                            : go(float{}, std::integral_constant<int, 64>{});
}

hga_status hga_gather_history(const hga_params* p, int64_t q_start, int64_t n_q, int64_t t_cap,
                              int64_t t_hist, const int32_t* group_idx, const int32_t* group_cnt,
                              const void* k_host, const void* v_host, void* k_dev, void* v_dev,
                              uint32_t* gen, uint32_t step, unsigned long long* bytes,
                              hga_stream_t stream) {
  hga::TierArgs a;
  hga_status s = tier_args(p, q_start, n_q, t_cap, t_hist, &a);
  if (s != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!group_idx || !group_cnt || !k_host || !v_host || !k_dev || !v_dev || !gen || step == 0)
    return HGA_ERR_INVALID_ARG;
  dim3 grid(a.n_blocks, a.Hkv);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto go = [&](auto tag, auto dim) {
    using T = decltype(tag);
    constexpr int D = decltype(dim)::value;
    return launch_pdl(hga::gather_history_kernel<D, T>, grid, dim3(256), 0, st, a, group_idx,
                      group_cnt, reinterpret_cast<const T*>(k_host),
                      reinterpret_cast<const T*>(v_host), reinterpret_cast<T*>(k_dev),
                      reinterpret_cast<T*>(v_dev), gen, step, bytes);
  };
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? go(__nv_bfloat16{}, std::integral_constant<int, 128>{})
                              : go(__nv_bfloat16{}, std::integral_constant<int, 64>{});
  return p->head_dim == 128 ? go(float{}, std::integral_constant<int, 128>{})
                            : go(float{}, std::integral_constant<int, 64>{});
}

hga_status hga_gather_store(const hga_params* p, const hga_kv_store* store, int64_t q_start,
                            int64_t n_q, int64_t t_hist, const int32_t* group_idx,
                            const int32_t* group_cnt, void* k_dev, void* v_dev, uint32_t* gen,
                            uint32_t step, unsigned long long* bytes, hga_stream_t stream) {
  if (!p || !store) return HGA_ERR_INVALID_ARG;
  hga::TierArgs a;
  hga_status s = tier_args(p, q_start, n_q, store->t_cap, t_hist, &a);
  if (s != HGA_OK) return s;
  if (p->n_kv_heads != store->Hkv || p->head_dim != store->d || p->dtype != store->dtype)
    return HGA_ERR_INVALID_ARG;
  if (t_hist > store->length) return HGA_ERR_INVALID_ARG;
  if (n_q == 0) return HGA_OK;
  if (!store->cache || !store->page_table || !group_idx || !group_cnt || !k_dev || !v_dev ||
      !gen || step == 0)
    return HGA_ERR_INVALID_ARG;
  hga::StoreArgs sa{store->cache, store->page_table, store->n_pages, store->page_tokens,
                    store->cache_pages, store->half_bytes};
  dim3 grid(a.n_blocks, a.Hkv);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto go = [&](auto tag, auto dim) {
    using T = decltype(tag);
    constexpr int D = decltype(dim)::value;
    return launch_pdl(hga::gather_store_kernel<D, T>, grid, dim3(256), 0, st, a, sa, group_idx,
                      group_cnt, reinterpret_cast<T*>(k_dev), reinterpret_cast<T*>(v_dev), gen,
                      step, bytes);
  };
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? go(__nv_bfloat16{}, std::integral_constant<int, 128>{})
                              : go(__nv_bfloat16{}, std::integral_constant<int, 64>{});
  return p->head_dim == 128 ? go(float{}, std::integral_constant<int, 128>{})
                            : go(float{}, std::integral_constant<int, 64>{});
}

hga_status hga_install_group_cache(const hga_params* p, int64_t t_cap,
                                   const void* group_sum_host, const hga_group_cache* cache,
                                   hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (t_cap <= 0 || !group_sum_host || !cache || !cache->data || !cache->tags || !cache->claims ||
      cache->cap <= 0 || cache->cap > 0x7fffffff)
    return HGA_ERR_INVALID_ARG;
  hga::TierArgs a{};
  a.Hkv = p->n_kv_heads;
  a.n_groups_cap = t_cap / p->group;
  a.cache_cap = cache->cap;
  const int64_t warps = (int64_t)a.Hkv * a.cache_cap;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffff) return HGA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto go = [&](auto tag, auto dim) {
    using T = decltype(tag);
    constexpr int D = decltype(dim)::value;
    return launch_pdl(hga::install_group_cache_kernel<D, T>, dim3((unsigned)blocks), dim3(256), 0,
                      st, a, reinterpret_cast<const T*>(group_sum_host),
                      reinterpret_cast<T*>(cache->data), cache->tags, cache->claims);
  };
  if (p->dtype == HGA_BF16)
    return p->head_dim == 128 ? go(__nv_bfloat16{}, std::integral_constant<int, 128>{})
                              : go(__nv_bfloat16{}, std::integral_constant<int, 64>{});
  return p->head_dim == 128 ? go(float{}, std::integral_constant<int, 128>{})
                            : go(float{}, std::integral_constant<int, 64>{});
}

hga_status hga_convert_v(const hga_params* p, const void* v, int64_t t_cap, int64_t t_begin,
                         int64_t t_end, void* v_f16, hga_stream_t stream) {
  hga_status s = check_params(p);
  if (s != HGA_OK) return s;
  if (p->dtype != HGA_BF16) return HGA_ERR_INVALID_ARG;
  if (t_cap <= 0 || t_begin < 0 || t_begin > t_end || t_end > t_cap) return HGA_ERR_INVALID_ARG;
  if (!v || !v_f16 || ((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(v_f16)) & 15))
    return HGA_ERR_INVALID_ARG;
  const char* vb = static_cast<const char*>(v);
  const char* ob = static_cast<const char*>(v_f16);
  const int64_t bytes = (int64_t)p->n_kv_heads * t_cap * p->head_dim * 2;
  if (vb != ob && vb < ob + bytes && ob < vb + bytes) return HGA_ERR_INVALID_ARG;
  if (t_begin == t_end) return HGA_OK;
  const int64_t n = (int64_t)p->n_kv_heads * (t_end - t_begin) * (p->head_dim / 8);
  const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto* src = static_cast<const __nv_bfloat16*>(v);
  auto* dst = static_cast<__half*>(v_f16);
  return p->head_dim == 128
             ? launch_pdl(hga::convert_v_kernel<128>, dim3(blocks), dim3(256), 0, st, src, dst,
                          t_cap, t_begin, t_end, p->n_kv_heads)
             : launch_pdl(hga::convert_v_kernel<64>, dim3(blocks), dim3(256), 0, st, src, dst,
                          t_cap, t_begin, t_end, p->n_kv_heads);
}

hga_status hga_selftest_exp2(const float* x, float* y, int64_t n, hga_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return HGA_ERR_INVALID_ARG;
  if (n == 0) return HGA_OK;
  const int64_t pairs = (n + 1) / 2;
  const unsigned blocks = (unsigned)std::min<int64_t>((pairs + 255) / 256, 1 << 20);
  hga::exp2_selftest_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return after_launch();
}

hga_status hga_set_kernel_variant(int32_t variant) {
  if (variant < 0 || variant > 2) return HGA_ERR_INVALID_ARG;
  g_kernel_variant.store(variant, std::memory_order_relaxed);
  return HGA_OK;
}

const char* hga_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

hga_status hga_set_wait_limit_ns(uint64_t ns) {
  if (ns < 1000000ull || ns > 60000000000ull) return HGA_ERR_INVALID_ARG;
  const unsigned long long v = ns;
  return cuda_ok(cudaMemcpyToSymbol(hga::g_wait_limit_ns, &v, sizeof(v)));
}

hga_status hga_selftest_wait(unsigned long long* elapsed_ns, hga_stream_t stream) {
  if (!elapsed_ns || (reinterpret_cast<uintptr_t>(elapsed_ns) & 7)) return HGA_ERR_INVALID_ARG;
  hga::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(elapsed_ns);
  return after_launch();
}

hga_status hga_debug_stall_next_attend(int64_t load_index) {
  if (load_index < -1) return HGA_ERR_INVALID_ARG;
  g_stall_next_attend.store(load_index, std::memory_order_relaxed);
  return HGA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of the history gather (see noalloc.cuh for which
// callers need it).  The stamps live in hga::g_static_gen; its device address
// is looked up once per device, with that device current, the first time the
// call runs there.
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_gen_mu;
uint32_t* g_static_gen_ptr[kMaxDevices] = {};

hga_status static_gen_address(cudaStream_t st, uint32_t** out) {
  int dev = -1;
  hga_status s = cuda_ok(cudaGetDevice(&dev));
  if (s != HGA_OK) return s;
  if (dev < 0 || dev >= kMaxDevices) return HGA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_gen_mu);
  if (!g_static_gen_ptr[dev]) {
    // The lookup may load the module; it is not done while `st` is being
    // captured into a graph.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if ((s = cuda_ok(cudaStreamIsCapturing(st, &cs))) != HGA_OK) return s;
    if (cs != cudaStreamCaptureStatusNone) return HGA_ERR_UNSUPPORTED;
    void* ptr = nullptr;
    if ((s = cuda_ok(cudaGetSymbolAddress(&ptr, hga::g_static_gen))) != HGA_OK) return s;
    g_static_gen_ptr[dev] = static_cast<uint32_t*>(ptr);
  }
  *out = g_static_gen_ptr[dev];
  return HGA_OK;
}

}  // namespace

extern "C" {

hga_status hga_gather_history_noalloc(const hga_params* p, int64_t q_start, int64_t n_q,
                                      int64_t t_cap, int64_t t_hist, const int32_t* group_idx,
                                      const int32_t* group_cnt, const void* k_host,
                                      const void* v_host, void* k_dev, void* v_dev,
                                      unsigned long long* bytes, hga_stream_t stream) {
  hga::TierArgs a;
  hga_status s = tier_args(p, q_start, n_q, t_cap, t_hist, &a);
  if (s != HGA_OK) return s;
  if (n_q == 0) return HGA_OK;
  if (!group_idx || !group_cnt || !k_host || !v_host || !k_dev || !v_dev)
    return HGA_ERR_INVALID_ARG;
  const int64_t words = (int64_t)a.Hkv * a.n_groups_cap;
  if (words > hga::kStaticGenWords) return HGA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* gen = nullptr;
  if ((s = static_gen_address(st, &gen)) != HGA_OK) return s;
  // Stamps left by an earlier call would read as "already copied": clear the
  // range this call uses, then gather with stamp 1.
  const unsigned blocks = (unsigned)std::min<int64_t>((words + 255) / 256, 148 * 8);
  hga::clear_stamps_kernel<<<blocks, 256, 0, st>>>(gen, words);
  if ((s = after_launch()) != HGA_OK) return s;
  return hga_gather_history(p, q_start, n_q, t_cap, t_hist, group_idx, group_cnt, k_host,
                            v_host, k_dev, v_dev, gen, 1u, bytes, stream);
}

}  // extern "C"
