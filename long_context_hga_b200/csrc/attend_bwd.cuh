// Backward of step 4: gradients of the gathered exact-token attention with the
// routing held fixed (the kept groups of every (query block, KV head) come
// from the forward pass and are inputs here).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: the attention
// reads exact token K/V of the kept groups plus the sink and local windows;
// the selection itself is piecewise constant, so gradients reach q, k and v
// only through that attention.  For a query row with attended set R:
//     s_j = q . k_j / sqrt(d),   p_j = exp(s_j - lse),   o = sum_j p_j v_j
//     dp_j = dO . v_j,   D = dO . o,   ds_j = p_j (dp_j - D)
//     dq = sum_j ds_j k_j / sqrt(d),  dk_j += ds_j q / sqrt(d),  dv_j += p_j dO
// with lse and o the forward's outputs (as given by the caller).
//
// First version, parity first: fp32 arithmetic on the CUDA cores.  One CTA
// per 128-row slice of a unit holds the slice's q, dO (fp32) in shared
// memory, walks the unit's group list one 8-token group at a time, keeps dq in
// registers and adds each group's dk, dv (summed over the slice's rows) to
// global memory with 16-byte fp32 atomics.  The products are dense
// contractions and belong on the tensor cores in a later version.
#pragma once
#include "attend.cuh"

namespace hga {

constexpr int kBwRows = 128;               // query rows per CTA
constexpr int kBwThreads = 256;

struct BwArgs {
  AttendArgs a;
  const void* o;       // [n_q][Hq][D], dtype of q
  const void* d_o;     // [n_q][Hq][D], dtype of q
  const float* lse;    // [n_q][Hq], natural log
  float* d_q;          // [n_q][Hq][D]
  float* d_k;          // [Hkv][t_cap][D]
  float* d_v;
  float scale;         // 1 / sqrt(D)
};

template <int D>
struct BwLayout {
  static constexpr int kStride = D + 4;   // padded rows, 16-byte aligned: float4 loads without bank conflicts
  static constexpr int kQ = 0;                                        // [128][D+1]
  static constexpr int kDO = kQ + kBwRows * kStride * 4;              // [128][D+1]
  static constexpr int kK = kDO + kBwRows * kStride * 4;              // [8][D+1]
  static constexpr int kV = kK + 8 * kStride * 4;                     // [8][D+1]
  static constexpr int kP = kV + 8 * kStride * 4;                     // [128][8]
  static constexpr int kDS = kP + kBwRows * 8 * 4;                    // [128][8]
  static constexpr int kRow = kDS + kBwRows * 8 * 4;                  // lse, D, pos
  static constexpr int kList = kRow + 3 * kBwRows * 4;
  static constexpr size_t smem_bytes(int max_list) { return (size_t)kList + (size_t)max_list * 4; }
};

template <typename E>
__device__ __forceinline__ float bw_load(const E* p);
template <>
__device__ __forceinline__ float bw_load<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float bw_load<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename E, int D>
__global__ void __launch_bounds__(kBwThreads) attend_bwd_kernel(BwArgs w) {
  using L = BwLayout<D>;
  constexpr int S = L::kStride;
  extern __shared__ __align__(128) char smem[];
  float* sq = reinterpret_cast<float*>(smem + L::kQ);
  float* sdo = reinterpret_cast<float*>(smem + L::kDO);
  float* sk = reinterpret_cast<float*>(smem + L::kK);
  float* sv = reinterpret_cast<float*>(smem + L::kV);
  float* sp = reinterpret_cast<float*>(smem + L::kP);
  float* sds = reinterpret_cast<float*>(smem + L::kDS);
  float* s_lse = reinterpret_cast<float*>(smem + L::kRow);
  float* s_d = s_lse + kBwRows;
  int* s_pos = reinterpret_cast<int*>(s_d + kBwRows);
  int* list = reinterpret_cast<int*>(smem + L::kList);
  const AttendArgs& a = w.a;

  griddep_wait();
  const int tid = threadIdx.x;
  const int b = blockIdx.y, h = blockIdx.z;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  const int row0 = blockIdx.x * kBwRows;
  if (row0 >= nrows) return;

  int n_nondiag;
  bool inv = false;
  const int n_list = build_group_list(a, b, h, b0, T, list, &n_nondiag, &inv);
  if (n_list < 0) return;

  // ---- the slice's rows: q, dO (fp32), lse, D = dO . o, position
  const E* q = static_cast<const E*>(a.q);
  const E* o = static_cast<const E*>(w.o);
  const E* d_o = static_cast<const E*>(w.d_o);
  for (int r = tid / 32; r < kBwRows; r += kBwThreads / 32) {
    const int lane = tid & 31;
    const int ur = row0 + r;
    const bool live = ur < nrows;
    const int64_t pos = b0 + (live ? ur / a.G : 0);
    const int64_t off = ((pos - a.q_start) * a.Hq + (int64_t)h * a.G + (live ? ur % a.G : 0)) * D;
    float dsum = 0.f;
    for (int c = lane; c < D; c += 32) {
      const float qv = live ? bw_load<E>(q + off + c) : 0.f;
      const float gv = live ? bw_load<E>(d_o + off + c) : 0.f;
      const float ov = live ? bw_load<E>(o + off + c) : 0.f;
      sq[r * S + c] = qv;
      sdo[r * S + c] = gv;
      dsum += gv * ov;
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, x);
    if (lane == 0) {
      s_d[r] = dsum;
      s_lse[r] = live ? w.lse[(pos - a.q_start) * a.Hq + (int64_t)h * a.G + ur % a.G] : 0.f;
      s_pos[r] = live ? (int)pos : -1;    // -1: no token is attended
    }
  }
  __syncthreads();

  // dq accumulators: row tid/2, columns [64 (tid%2), 64 (tid%2) + 64)
  constexpr int kHalfD = D / 2;
  float dq[kHalfD];
#pragma unroll
  for (int c = 0; c < kHalfD; ++c) dq[c] = 0.f;
  const int rq = tid >> 1, cq = (tid & 1) * kHalfD;
  const E* kh = static_cast<const E*>(a.k) + (int64_t)h * a.t_cap * D;
  const E* vh = static_cast<const E*>(a.v) + (int64_t)h * a.t_cap * D;

  // K/V of one 8-token group, kPer elements of each per thread; the next
  // group's loads are issued before the current group's products so that
  // their latency hides behind them (tokens at or past T, and skipped
  // entries, read as zero and are never attended)
  constexpr int kPer = 8 * D / kBwThreads;
  static_assert(8 * D % kBwThreads == 0, "K/V elements per thread");
  float kreg[kPer], vreg[kPer];
  auto fetch = [&](int li) {
    const int ent = li < n_list ? list[li] : -1;
    const int64_t g0 = (int64_t)ent * a.group;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int x = tid + i * kBwThreads, j = x / D, c = x % D;
      const bool in = ent >= 0 && g0 + j < T;
      kreg[i] = in ? bw_load<E>(kh + (g0 + j) * D + c) : 0.f;
      vreg[i] = in ? bw_load<E>(vh + (g0 + j) * D + c) : 0.f;
    }
  };
  fetch(0);
  for (int li = 0; li < n_list; ++li) {
    const int ent = list[li];                     // uniform; < 0: skipped entry
    const int64_t t0 = (int64_t)ent * a.group;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int x = tid + i * kBwThreads, j = x / D, c = x % D;
      sk[j * S + c] = kreg[i];
      sv[j * S + c] = vreg[i];
    }
    __syncthreads();
    fetch(li + 1);
    if (ent < 0) {
      __syncthreads();                            // no products for a skipped entry
      continue;
    }
    // ---- p and ds for (row tid/2, tokens 4 (tid%2) .. +4): register tile
    // of 4 dot products of each kind, 16-byte shared loads along d
    {
      const int r = tid >> 1, j0 = (tid & 1) * 4;
      const int pos = s_pos[r];
      float sv4[4] = {0.f, 0.f, 0.f, 0.f}, dp4[4] = {0.f, 0.f, 0.f, 0.f};
      const float4* qr = reinterpret_cast<const float4*>(sq + r * S);
      const float4* gr = reinterpret_cast<const float4*>(sdo + r * S);
#pragma unroll 4
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 x = qr[c4], g = gr[c4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float4 kk = reinterpret_cast<const float4*>(sk + (j0 + jj) * S)[c4];
          const float4 vv = reinterpret_cast<const float4*>(sv + (j0 + jj) * S)[c4];
          sv4[jj] = fmaf(x.x, kk.x, fmaf(x.y, kk.y, fmaf(x.z, kk.z, fmaf(x.w, kk.w, sv4[jj]))));
          dp4[jj] = fmaf(g.x, vv.x, fmaf(g.y, vv.y, fmaf(g.z, vv.z, fmaf(g.w, vv.w, dp4[jj]))));
        }
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = j0 + jj;
        const bool valid = pos >= 0 && t0 + j <= pos;
        const float p = valid ? expf(sv4[jj] * w.scale - s_lse[r]) : 0.f;
        sp[r * 8 + j] = p;
        sds[r * 8 + j] = valid ? p * (dp4[jj] - s_d[r]) : 0.f;
      }
    }
    __syncthreads();
    // ---- dq (registers) for row tid/2, half tid%2 of the columns
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float ds = sds[rq * 8 + j] * w.scale;
      const float4* kr = reinterpret_cast<const float4*>(sk + j * S + cq);
#pragma unroll
      for (int c4 = 0; c4 < kHalfD / 4; ++c4) {
        const float4 kk = kr[c4];
        dq[4 * c4] = fmaf(ds, kk.x, dq[4 * c4]);
        dq[4 * c4 + 1] = fmaf(ds, kk.y, dq[4 * c4 + 1]);
        dq[4 * c4 + 2] = fmaf(ds, kk.z, dq[4 * c4 + 2]);
        dq[4 * c4 + 3] = fmaf(ds, kk.w, dq[4 * c4 + 3]);
      }
    }
    // ---- dk, dv of token tid/32, columns 4 (tid%32) .. +4, summed over rows
    {
      const int j = tid >> 5, c0 = (tid & 31) * 4;
      if (c0 < D && t0 + j < T) {
        float4 dk = make_float4(0.f, 0.f, 0.f, 0.f), dv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int r = 0; r < kBwRows; ++r) {
          const float ds = sds[r * 8 + j], p = sp[r * 8 + j];
          const float4 qr = *reinterpret_cast<const float4*>(sq + r * S + c0);
          const float4 gr = *reinterpret_cast<const float4*>(sdo + r * S + c0);
          dk.x = fmaf(ds, qr.x, dk.x); dk.y = fmaf(ds, qr.y, dk.y);
          dk.z = fmaf(ds, qr.z, dk.z); dk.w = fmaf(ds, qr.w, dk.w);
          dv.x = fmaf(p, gr.x, dv.x); dv.y = fmaf(p, gr.y, dv.y);
          dv.z = fmaf(p, gr.z, dv.z); dv.w = fmaf(p, gr.w, dv.w);
        }
        dk.x *= w.scale; dk.y *= w.scale; dk.z *= w.scale; dk.w *= w.scale;
        const int64_t off = ((int64_t)h * a.t_cap + t0 + j) * D + c0;
        atomicAdd(reinterpret_cast<float4*>(w.d_k + off), dk);
        atomicAdd(reinterpret_cast<float4*>(w.d_v + off), dv);
      }
    }
    __syncthreads();                              // before the next group's K/V
  }

  // ---- dq of the live rows
  const int ur = row0 + rq;
  if (ur < nrows) {
    const int64_t pos = b0 + ur / a.G;
    float* dst = w.d_q + ((pos - a.q_start) * a.Hq + (int64_t)h * a.G + ur % a.G) * D + cq;
#pragma unroll
    for (int c = 0; c < kHalfD; c += 4)
      *reinterpret_cast<float4*>(dst + c) = make_float4(dq[c], dq[c + 1], dq[c + 2], dq[c + 3]);
  }
  griddep_launch();
}

}  // namespace hga
