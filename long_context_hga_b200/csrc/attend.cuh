// Step 4: exact-token attention over the routed set.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: only the exact
// token K/V of the selected groups enter the routed working set, besides the
// fixed sink and local windows; summaries are never values.  Attention is
// causal softmax attention.
//
// Per (query block b, KV head h) the attended tokens form a list of 8-token
// groups: sink groups, routed groups (ascending), local-window groups, then the
// block's own diagonal groups.  In the head-major K/V layout each group is one
// contiguous 8 x d span, so a 64-token K/V tile is 8 independent 2 KB (d=128)
// copies.  Rows of a unit are (position, query head) pairs, position-major, so
// the G query heads sharing the KV head reuse every gathered tile (GQA
// packing).  This file holds the portable mma.sync variant (FA2-style, one
// warp per 16 rows, P kept in registers) and the exact FFMA fp32 variant.
#pragma once
#include "common.cuh"
#include "route.cuh"

namespace hga {

struct AttendArgs {
  const void* q;          // [n_q][Hq][D]
  const void* k;          // [Hkv][t_cap][D]
  const void* v;
  int64_t q_start, n_q, t_cap;
  const int32_t* group_idx;  // [Hkv][n_blocks][cap_g]
  const int32_t* group_cnt;
  int64_t cap_g;
  void* o;
  float* lse;
  int n_blocks, Hq, Hkv, G;
  int group, qblock, sink, local;
  int max_list;           // group-list slots in shared memory
  int64_t pos_lo;         // rows of positions before pos_lo may be skipped (their
                          // outputs left as they are); q_start computes every row
  float scale_log2;       // log2(e) / sqrt(d)
  int q_early;            // q may be requested before waiting for the previous kernel
};

// Builds the unit's group list in shared memory; returns the entry count and
// the number of entries before the diagonal.  Invalid routed entries become -1
// (skipped) and are reported.
__device__ __forceinline__ int build_group_list(const AttendArgs& a, int b, int h, int64_t b0,
                                                int64_t T, int* list, int* n_nondiag,
                                                bool* any_invalid) {
  const int g = a.group;
  const int64_t sink_end = min((int64_t)a.sink, b0);
  const int n_s = (int)(sink_end / g);
  int n_r = a.group_cnt[(int64_t)h * a.n_blocks + b];
  const int32_t* routed = a.group_idx + ((int64_t)h * a.n_blocks + b) * a.cap_g;
  const int64_t loc_lo = max(sink_end, b0 - a.local);
  const int n_l = (int)((b0 - loc_lo) / g);
  const int64_t b_end = min(b0 + a.qblock, T);
  const int n_d = (int)((b_end - b0 + g - 1) / g);
  bool bad = false;
  if (n_r < 0 || n_r > a.cap_g) { bad = true; n_r = 0; }
  const int n = n_s + n_r + n_l + n_d;
  if (n > a.max_list) { if (threadIdx.x == 0) report(HGA_ERR_DEVICE_CHECK); return -1; }
  const int64_t lo_tok = a.sink, hi_tok = b0 - a.local;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    int e;
    if (i < n_s) e = i;
    else if (i < n_s + n_r) {
      const int r = i - n_s;
      e = routed[r];
      const bool ok = (int64_t)e * g >= lo_tok && ((int64_t)e + 1) * g <= hi_tok &&
                      (r == 0 || e > routed[r - 1]);
      if (!ok) { e = -1; bad = true; }
    } else if (i < n_s + n_r + n_l) e = (int)(loc_lo / g) + (i - n_s - n_r);
    else e = (int)(b0 / g) + (i - n_s - n_r - n_l);
    list[i] = e;
  }
  if (bad) { report(HGA_ERR_DEVICE_CHECK); *any_invalid = true; }
  *n_nondiag = n_s + n_r + n_l;
  return n;
}

// Converts n16 16-byte chunks of bf16 at `tile` (shared memory) to fp16 in
// place, cooperatively over `nthreads` threads.  bf16 -> fp16 is exact for
// 2^-14 <= |x| < 65504 (8 significant bits fit in 11) and loses at most 2^-25
// below; a finite value that overflows fp16 is reported (HGA_ERR_DEVICE_CHECK).
__device__ __forceinline__ void convert_tile_bf16_to_f16(char* tile, int n16, int nthreads) {
  bool overflow = false;
  for (int i = threadIdx.x; i < n16; i += nthreads) {
    uint4 raw = *reinterpret_cast<const uint4*>(tile + i * 16);
    uint32_t* w = reinterpret_cast<uint32_t*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      overflow |= (fabsf(f.x) > 65504.f) | (fabsf(f.y) > 65504.f);
      __half2 hv = __floats2half2_rn(f.x, f.y);
      w[j] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    *reinterpret_cast<uint4*>(tile + i * 16) = raw;
  }
  if (overflow) report(HGA_ERR_DEVICE_CHECK);
}

// ---------------------------------------------------------------- bf16, mma.sync

constexpr int kAttRows = 64;      // rows per CTA (4 warps x 16)
constexpr int kAttTok = 64;       // tokens per K/V tile (8 groups)

// VF16: V is already fp16 in memory (no per-tile conversion).
template <int D, bool VF16 = false>
__global__ void __launch_bounds__(128) attend_mma_kernel(AttendArgs a) {
  extern __shared__ __align__(128) char smem[];
  char* sq = smem;                                  // [64][D] bf16, swizzled
  char* sk = sq + kAttRows * D * 2;                 // [2][64][D]
  char* sv = sk + 2 * kAttTok * D * 2;              // [2][64][D]
  int* list = reinterpret_cast<int*>(sv + 2 * kAttTok * D * 2);
  __shared__ bool s_invalid;

  griddep_wait();
  const int tile_r = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  const int r0 = tile_r * kAttRows;
  if (r0 >= nrows) return;
  if (tid == 0) s_invalid = false;
  __syncthreads();
  int n_nondiag;
  bool inv = false;
  const int n_list = build_group_list(a, b, h, b0, T, list, &n_nondiag, &inv);
  if (n_list < 0) return;
  if (inv) s_invalid = true;

  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kh = reinterpret_cast<const __nv_bfloat16*>(a.k) + (int64_t)h * a.t_cap * D;
  const __nv_bfloat16* vh = reinterpret_cast<const __nv_bfloat16*>(a.v) + (int64_t)h * a.t_cap * D;
  const int64_t row_stride = (int64_t)a.Hq * D;
  const __nv_bfloat16* qblk = q + (b0 - a.q_start) * row_stride + (int64_t)h * a.G * D;
  constexpr int kCh = D / 8;

  // stage Q rows (zero past the unit's rows)
  for (int e = tid; e < kAttRows * kCh; e += 128) {
    const int r = e / kCh, ch = e % kCh, rr = r0 + r;
    const bool ok = rr < nrows;
    const __nv_bfloat16* src = qblk + (int64_t)(ok ? rr / a.G : 0) * row_stride + (ok ? rr % a.G : 0) * D + ch * 8;
    cp_async16(smem_u32(sq + swz<D>(r, ch)), src, ok ? 16 : 0);
  }
  __syncthreads();   // list visible
  const int n_tiles = (n_list + 7) / 8;
  auto load_kv = [&](int t, int buf) {
    char* dk = sk + buf * (kAttTok * D * 2);
    char* dv = sv + buf * (kAttTok * D * 2);
    for (int e = tid; e < kAttTok * kCh; e += 128) {
      const int r = e / kCh, ch = e % kCh;
      const int li = t * 8 + (r >> 3);
      const int ent = li < n_list ? list[li] : -1;
      const int64_t tok = (int64_t)ent * a.group + (r & 7);
      const bool ok = ent >= 0 && tok < T;
      const int64_t off = (ok ? tok : 0) * D + ch * 8;
      cp_async16(smem_u32(dk + swz<D>(r, ch)), kh + off, ok ? 16 : 0);
      cp_async16(smem_u32(dv + swz<D>(r, ch)), vh + off, ok ? 16 : 0);
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  // per-thread rows: g and g+8 of this warp's 16
  const int g = lane >> 2, tq = lane & 3;
  const int row_a = r0 + warp * 16 + g, row_b = row_a + 8;
  const int64_t pos_a = b0 + row_a / a.G, pos_b = b0 + row_b / a.G;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) oacc[i][j] = 0.f;
  uint32_t qf[D / 16][4];
  const bool need_mask_all = s_invalid;

  for (int t = 0; t < n_tiles; ++t) {
    if (t + 1 < n_tiles) load_kv(t + 1, (t + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldsm_x4(smem_u32(sq + swz<D>(r, ch)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const char* tk = sk + (t & 1) * (kAttTok * D * 2);
    const char* tv = sv + (t & 1) * (kAttTok * D * 2);
    // V tile bf16 -> fp16 in place (exact for |v| < 65504; larger is reported)
    if constexpr (!VF16)
      convert_tile_bf16_to_f16(sv + (t & 1) * (kAttTok * D * 2), kAttTok * D / 8, 128);
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[nt][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0r, b1r, b2r, b3r;
        ldsm_x4(smem_u32(tk + swz<D>(r, ch)), b0r, b1r, b2r, b3r);
        mma_bf16(s[2 * np], qf[kk], b0r, b1r);
        mma_bf16(s[2 * np + 1], qf[kk], b2r, b3r);
      }
    }
    // mask: padding entries, invalid routed entries, causal diagonal
    const bool need_mask = need_mask_all || (t * 8 + 8 > n_nondiag);
    if (need_mask) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int li = t * 8 + nt;
        const int ent = li < n_list ? list[li] : -1;
        const int64_t tok0 = (int64_t)ent * a.group + 2 * tq;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int64_t tok = tok0 + j;
          const bool okt = ent >= 0;
          if (!(okt && tok <= pos_a)) s[nt][j] = -INFINITY;
          if (!(okt && tok <= pos_b)) s[nt][2 + j] = -INFINITY;
        }
      }
    }
    // online softmax (base 2)
    float mx_a = m_a, mx_b = m_b;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]) * a.scale_log2);
      mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]) * a.scale_log2);
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float use_a = mx_a == -INFINITY ? 0.f : mx_a;
    const float use_b = mx_b == -INFINITY ? 0.f : mx_b;
    const float corr_a = exp2f(m_a - use_a), corr_b = exp2f(m_b - use_b);
    m_a = mx_a;
    m_b = mx_b;
    float sum_a = 0.f, sum_b = 0.f;
    uint32_t pf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = exp2f(s[nt][0] * a.scale_log2 - use_a);
      const float p1 = exp2f(s[nt][1] * a.scale_log2 - use_a);
      const float p2 = exp2f(s[nt][2] * a.scale_log2 - use_b);
      const float p3 = exp2f(s[nt][3] * a.scale_log2 - use_b);
      sum_a += p0 + p1;
      sum_b += p2 + p3;
      __half2 lo = __floats2half2_rn(p0, p1);
      __half2 hi = __floats2half2_rn(p2, p3);
      pf[nt >> 1][(nt & 1) * 2 + 0] = *reinterpret_cast<uint32_t*>(&lo);
      pf[nt >> 1][(nt & 1) * 2 + 1] = *reinterpret_cast<uint32_t*>(&hi);
    }
    l_a = l_a * corr_a + sum_a;
    l_b = l_b * corr_b + sum_b;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      oacc[nd][0] *= corr_a;
      oacc[nd][1] *= corr_a;
      oacc[nd][2] *= corr_b;
      oacc[nd][3] *= corr_b;
    }
    // O += P V in fp16 x fp16 -> fp32 (A = P from registers: a0 = rows g /
    // tokens 2t of n-tile 2kk, ...).  P in [0, 1] keeps 11 significant bits in
    // fp16 against 8 in bf16.
    __syncthreads();   // converted V tile visible
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t af[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
      for (int nd2 = 0; nd2 < D / 16; ++nd2) {
        const int r = kk * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int ch = nd2 * 2 + (lane >> 4);
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(smem_u32(tv + swz<D>(r, ch)), v0, v1, v2, v3);
        mma_f16(oacc[2 * nd2], af, v0, v1);
        mma_f16(oacc[2 * nd2 + 1], af, v2, v3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // row sums across the quad
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = 1.f / l_a, inv_b = 1.f / l_b;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.o);
  const int64_t hq_a = (int64_t)h * a.G + row_a % a.G, hq_b = (int64_t)h * a.G + row_b % a.G;
  if (row_a < nrows) {
    __nv_bfloat16* dst = o + ((pos_a - a.q_start) * a.Hq + hq_a) * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
      *reinterpret_cast<__nv_bfloat162*>(dst + nd * 8 + 2 * tq) =
          __floats2bfloat162_rn(oacc[nd][0] * inv_a, oacc[nd][1] * inv_a);
    if (a.lse && tq == 0)
      a.lse[(pos_a - a.q_start) * a.Hq + hq_a] = (m_a + log2f(l_a)) * 0.6931471805599453f;
  }
  if (row_b < nrows) {
    __nv_bfloat16* dst = o + ((pos_b - a.q_start) * a.Hq + hq_b) * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
      *reinterpret_cast<__nv_bfloat162*>(dst + nd * 8 + 2 * tq) =
          __floats2bfloat162_rn(oacc[nd][2] * inv_b, oacc[nd][3] * inv_b);
    if (a.lse && tq == 0)
      a.lse[(pos_b - a.q_start) * a.Hq + hq_b] = (m_b + log2f(l_b)) * 0.6931471805599453f;
  }
}

template <int D>
inline size_t attend_mma_smem_bytes(int max_list) {
  return (size_t)kAttRows * D * 2 + 4 * (size_t)kAttTok * D * 2 + (size_t)max_list * 4;
}

// ---------------------------------------------------------------- fp32, FFMA

constexpr int kAttF32Rows = 8;   // one warp per row

template <int D>
__global__ void __launch_bounds__(256) attend_f32_kernel(AttendArgs a) {
  extern __shared__ __align__(128) char smem[];
  int* list = reinterpret_cast<int*>(smem);
  __shared__ bool s_invalid;
  griddep_wait();
  const int tile_r = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  if (tile_r * kAttF32Rows >= nrows) return;
  if (threadIdx.x == 0) s_invalid = false;
  __syncthreads();
  int n_nondiag;
  bool inv = false;
  const int n_list = build_group_list(a, b, h, b0, T, list, &n_nondiag, &inv);
  if (n_list < 0) return;
  __syncthreads();
  const int row = tile_r * kAttF32Rows + warp;
  if (row >= nrows) return;
  const int64_t pos = b0 + row / a.G;
  const int64_t hq = (int64_t)h * a.G + row % a.G;
  const float* qv = reinterpret_cast<const float*>(a.q) + ((pos - a.q_start) * a.Hq + hq) * D;
  const float* kh = reinterpret_cast<const float*>(a.k) + (int64_t)h * a.t_cap * D;
  const float* vh = reinterpret_cast<const float*>(a.v) + (int64_t)h * a.t_cap * D;
  constexpr int kPer = D / 32;
  float qr[kPer], acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) { qr[i] = qv[lane + 32 * i]; acc[i] = 0.f; }
  float m = -INFINITY, l = 0.f;
  for (int li = 0; li < n_list; ++li) {
    const int ent = list[li];
    if (ent < 0) continue;
    for (int j = 0; j < a.group; ++j) {
      const int64_t tok = (int64_t)ent * a.group + j;
      if (tok > pos) break;
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) d = fmaf(qr[i], kh[tok * D + lane + 32 * i], d);
      d = warp_sum(d) * a.scale_log2;
      const float mn = fmaxf(m, d);
      const float corr = exp2f(m - mn), p = exp2f(d - mn);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] = acc[i] * corr + p * vh[tok * D + lane + 32 * i];
      m = mn;
    }
  }
  float* o = reinterpret_cast<float*>(a.o) + ((pos - a.q_start) * a.Hq + hq) * D;
#pragma unroll
  for (int i = 0; i < kPer; ++i) o[lane + 32 * i] = acc[i] / l;
  if (a.lse && lane == 0) a.lse[(pos - a.q_start) * a.Hq + hq] = (m + log2f(l)) * 0.6931471805599453f;
}

}  // namespace hga
