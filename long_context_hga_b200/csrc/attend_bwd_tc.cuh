// Backward of step 4 on the sm_100a tensor cores (bf16 inputs): gradients of
// the gathered exact-token attention with the routing held fixed.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: the routed
// attention is exact-token softmax attention over the kept groups plus the
// sink and local windows, and training differentiates through it (section
// 2.2); the selection is piecewise constant and passes no gradient.  For a
// query row with attended set R (s_j = q.k_j/sqrt(d), p_j = exp(s_j - lse)):
//     dp_j = dO.v_j,  D = dO.o,  ds_j = p_j (dp_j - D)
//     dq = sum_j ds_j k_j / sqrt(d),  dk_j += ds_j q / sqrt(d),  dv_j += p_j dO
//
// Three launches, each a dense contraction on tcgen05 where there is one:
//   bwd_dsum_kernel   D = rowsum(dO * o) per query row (fp32), written to
//                     column 0 of the row of d_q (d_q is output only; the dQ
//                     kernel reads each row's D before it writes that row)
//   bwd_dkdv_kernel   one CTA per (K/V tile of 128 tokens, unit): for every
//                     128-row tile of the unit's rows
//                       S^T = K Q^T, dP^T = V dO^T  (M = tokens, N = rows)
//                       P^T, dS^T (bf16) written over S^T, dP^T in TMEM
//                       dV += P^T dO, dK += dS^T Q  (TMEM accumulators)
//                     then one float4 atomic add per 4 values of the tile's
//                     dK, dV rows (tokens shared by several units, e.g. the
//                     sink, receive one add per unit)
//   bwd_dq_kernel     one CTA per 128-row tile of a unit: for every K/V tile
//                       S = Q K^T, dP = dO V^T  (M = rows, N = tokens)
//                       dS (bf16) written over S in TMEM
//                       dQ += dS K              (TMEM accumulator)
//                     then dQ stored once
// P and dS are rounded to bf16 (8 significant bits) as MMA operands: both
// operands of one tcgen05.mma kind::f16 have the same type, and Q, dO, K are
// bf16.  Everything else accumulates in fp32.  Padding entries of a tile load
// a group past the end of the K/V tensor, which TMA fills with zeros, so no
// stale shared memory meets a zero weight.
#pragma once
#include "attend_bwd.cuh"
#include "attend_tc.cuh"

namespace hga {

constexpr int kBtRows = 128;              // rows per row tile
constexpr int kBtTok = 128;               // tokens per K/V tile
constexpr int kBtGroupsPerTile = kBtTok / 8;
constexpr int kBtThreads = 256;           // 0 producer, 1 MMA, 2-3 idle, 4-7 softmax
constexpr float kLog2e = 1.4426950408889634f;

struct BtArgs {
  AttendArgs a;
  const void* o;        // [n_q][Hq][D] bf16
  const void* d_o;      // [n_q][Hq][D] bf16
  const float* lse;     // [n_q][Hq], natural log
  float* d_q;           // [n_q][Hq][D]; column 0 holds D = dO.o on entry of the
                        // dK/dV and dQ kernels
  float* d_k;           // [Hkv][t_cap][D], accumulated
  float* d_v;
  float scale;          // 1 / sqrt(D)
  float scale_log2;     // log2(e) / sqrt(D)
};

// ---------------------------------------------------------------- D

// D = sum_c dO[row][c] * o[row][c] over all n_rows = n_q * Hq rows, one warp
// per row, 16-byte loads; written to d_q[row * Dh].
template <int Dh>
__global__ void __launch_bounds__(256) bwd_dsum_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ d_o,
                                                       float* __restrict__ d_q, int64_t n_rows) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; row < n_rows;
       row += warps) {
    float s = 0.f;
    if (lane < Dh / 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(o + row * Dh + lane * 8);
      const uint4 g = *reinterpret_cast<const uint4*>(d_o + row * Dh + lane * 8);
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&x);
      const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(xh[i]), b = __bfloat1622float2(gh[i]);
        s = fmaf(a.x, b.x, fmaf(a.y, b.y, s));
      }
    }
    s = warp_sum(s);
    if (lane == 0) d_q[row * Dh] = s;
  }
  griddep_launch();
}

// ---------------------------------------------------------------- shared

// Entry li of a unit's group list (sink, routed, local window, diagonal; the
// list build_group_list_tc makes), validated like it: a routed entry outside
// the routed range or not above its predecessor is -1.  n_r is the routed
// count as read (an out-of-range count counts as zero).
struct BtList {
  int n_s, n_r, n_l, n_list, n_nondiag;
  int64_t loc_lo_g, diag_g, lo_tok, hi_tok;
  const int32_t* routed;
};
__device__ __forceinline__ BtList bt_list(const AttendArgs& a, int b, int h, int64_t b0,
                                          int64_t T) {
  BtList L;
  const int g = a.group;
  const int64_t sink_end = min((int64_t)a.sink, b0);
  L.n_s = (int)(sink_end / g);
  L.n_r = a.group_cnt[(int64_t)h * a.n_blocks + b];
  if (L.n_r < 0 || L.n_r > a.cap_g) L.n_r = 0;
  const int64_t loc_lo = max(sink_end, b0 - a.local);
  L.n_l = (int)((b0 - loc_lo) / g);
  const int64_t b_end = min(b0 + a.qblock, T);
  L.n_nondiag = L.n_s + L.n_r + L.n_l;
  L.n_list = L.n_nondiag + (int)((b_end - b0 + g - 1) / g);
  L.loc_lo_g = loc_lo / g;
  L.diag_g = b0 / g;
  L.lo_tok = a.sink;
  L.hi_tok = b0 - a.local;
  L.routed = a.group_idx + ((int64_t)h * a.n_blocks + b) * a.cap_g;
  return L;
}
__device__ __forceinline__ int bt_entry(const BtList& L, int li, int g) {
  if (li < L.n_s) return li;
  if (li < L.n_s + L.n_r) {
    const int r = li - L.n_s;
    const int e = L.routed[r];
    const bool ok = (int64_t)e * g >= L.lo_tok && ((int64_t)e + 1) * g <= L.hi_tok &&
                    (r == 0 || e > L.routed[r - 1]);
    return ok ? e : -1;
  }
  if (li < L.n_nondiag) return (int)(L.loc_lo_g + (li - L.n_s - L.n_r));
  if (li < L.n_list) return (int)(L.diag_g + (li - L.n_nondiag));
  return -1;
}

// The 16 groups of one K/V tile into a [group][half][8 rows][128 B] buffer
// (producer warp; lane e < 16 owns entry e).  Eight aligned consecutive
// valid groups come as one box; an entry with no group loads the group past
// the end of the tensor, which TMA fills with zeros.  Every call moves
// 16 * halves * 1 KB bytes, counted on `bar`.
template <int D>
__device__ __forceinline__ void bt_load_tile(char* dst, const CUtensorMap* m1, const CUtensorMap* m8,
                                             int ent, int64_t head_group0, int zero_group,
                                             uint64_t* bar, int lane) {
  constexpr int kGroupBytes = (D / 64) * 1024;
  const int e = lane & 15;
  const int ent0 = __shfl_sync(0xffffffffu, ent, e & ~7);
  const bool consec = ent >= 0 && ent0 >= 0 && ent == ent0 + (e & 7);
  const unsigned cons_mask = __ballot_sync(0xffffffffu, lane < 16 && consec);
  const bool run = ((cons_mask >> (e & ~7)) & 0xffu) == 0xffu;
  if (lane < 16) {
    const int gcoord = ent >= 0 ? (int)(head_group0 + ent) : zero_group;
    if (run) {
      if ((e & 7) == 0) tc::tma_load_4d(dst + e * kGroupBytes, m8, 0, 0, 0, gcoord, bar);
    } else {
      tc::tma_load_4d(dst + e * kGroupBytes, m1, 0, 0, 0, gcoord, bar);
    }
  }
}

// ---------------------------------------------------------------- dK, dV

template <int D>
struct BtKvLayout {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kBtRows * 128;               // one 64-column half of 128 rows
  static constexpr int kRowTileBytes = kHalves * kHalfBytes;     // Q or dO of one row tile
  static constexpr int kGroupBytes = kHalves * 8 * 128;
  static constexpr int kTileBytes = kBtGroupsPerTile * kGroupBytes;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kStage = kV + kTileBytes;                 // [2][Q | dO]
  static constexpr int kRowVals = kStage + 2 * 2 * kRowTileBytes; // [2][lse | D][128] floats
  static constexpr int kBar = kRowVals + 2 * 2 * kBtRows * 4;
  static constexpr size_t smem_bytes() { return 1024 + (size_t)kBar + 256; }
};

struct BtKvBars {
  uint64_t kv_full, stage_full[2], stage_empty[2], sdp_full, p_full, acc_full, done;
  uint64_t rows_ready[2];   // lse / D of a row tile in shared memory (128 arrivals)
  uint32_t tmem_base;
  int abort;
};

template <int D>
__device__ __noinline__ void bt_kv_mma(BtKvBars* bars, uint32_t tmem, uint32_t k_base,
                                      uint32_t v_base, uint32_t stage_base, int n_rt,
                                      volatile int* abort_flag) {
  using L = BtKvLayout<D>;
  constexpr uint32_t kIdS = tc::idesc_f16(kBtTok, kBtRows, 1, 0);   // M tokens, N rows
  constexpr uint32_t kIdAcc = tc::idesc_f16(kBtTok, D, 1, 1);       // M tokens, N = d (MN-major B)
  const uint64_t k_desc = tc::sdesc_sw128(k_base, 16, L::kGroupBytes);
  const uint64_t v_desc = tc::sdesc_sw128(v_base, 16, L::kGroupBytes);
  bool ok = tc::mbar_wait_warp(&bars->kv_full, 0, abort_flag);
  for (int rt = 0; ok && rt < n_rt; ++rt) {
    const int s = rt & 1;
    if (!(ok = tc::mbar_wait_warp(&bars->stage_full[s], (rt >> 1) & 1, abort_flag))) break;
    tc::fence_after_sync();
    const uint32_t q_base = stage_base + s * 2 * L::kRowTileBytes;
    const uint32_t do_base = q_base + L::kRowTileBytes;
    const uint64_t q_kmaj = tc::sdesc_sw128(q_base, 16, 1024);
    const uint64_t do_kmaj = tc::sdesc_sw128(do_base, 16, 1024);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t ko = (uint32_t)(((k >> 2) * 1024 + (k & 3) * 32) >> 4);
      const uint32_t qo = (uint32_t)(((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4);
      tc::mma_ss_warp(tmem + 0, k_desc + ko, q_kmaj + qo, kIdS, k > 0);        // S^T
    }
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t ko = (uint32_t)(((k >> 2) * 1024 + (k & 3) * 32) >> 4);
      const uint32_t qo = (uint32_t)(((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4);
      tc::mma_ss_warp(tmem + 128, v_desc + ko, do_kmaj + qo, kIdS, k > 0);     // dP^T
    }
    tc::mma_commit_warp(&bars->sdp_full);
    if (!(ok = tc::mbar_wait_warp(&bars->p_full, rt & 1, abort_flag))) break;
    tc::fence_after_sync();
    // B = dO or Q as [rows (K)][d (N)], N contiguous: halves L::kHalfBytes
    // apart, 8-row chunks 1 KB apart; one K step of 16 rows is 2 KB
    const uint64_t do_mn = tc::sdesc_sw128(do_base, L::kHalfBytes, 1024);
    const uint64_t q_mn = tc::sdesc_sw128(q_base, L::kHalfBytes, 1024);
#pragma unroll
    for (int k = 0; k < kBtRows / 16; ++k)
      tc::mma_ts_warp(tmem + 256, tmem + 0 + k * 8, do_mn + (uint64_t)((k * 2048) >> 4), kIdAcc,
                      (rt > 0 || k > 0) ? 1u : 0u);                        // dV += P^T dO
#pragma unroll
    for (int k = 0; k < kBtRows / 16; ++k)
      tc::mma_ts_warp(tmem + 384, tmem + 128 + k * 8, q_mn + (uint64_t)((k * 2048) >> 4), kIdAcc,
                      (rt > 0 || k > 0) ? 1u : 0u);                        // dK += dS^T Q
    tc::mma_commit_warp(&bars->stage_empty[s]);
  }
  tc::mma_commit_warp(&bars->acc_full);
  tc::mma_commit_warp(&bars->done);
  const uint64_t t0 = tc::globaltimer_ns();
  while (!tc::mbar_try_wait(&bars->done, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
  }
}

template <int D>
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k1,
                    const __grid_constant__ CUtensorMap tm_k8,
                    const __grid_constant__ CUtensorMap tm_v1,
                    const __grid_constant__ CUtensorMap tm_v8, BtArgs w) {
  using L = BtKvLayout<D>;
  const AttendArgs& a = w.a;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BtKvBars* bars = reinterpret_cast<BtKvBars*>(smem + L::kBar);
  float* rowvals = reinterpret_cast<float*>(smem + L::kRowVals);   // [2][lse_log2 | D][128]
  volatile int* abort_flag = &bars->abort;

  griddep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int jt = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  const int n_rt = (nrows + kBtRows - 1) / kBtRows;
  const BtList lst = bt_list(a, b, h, b0, T);
  if (jt * kBtGroupsPerTile >= lst.n_list) return;      // uniform: this unit has fewer tiles

  if (tid == 0) {
    bars->abort = 0;
    tc::mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->stage_full[s], 1);
      tc::mbar_init(&bars->stage_empty[s], 1);
    }
    tc::mbar_init(&bars->sdp_full, 1);
    tc::mbar_init(&bars->p_full, kBtRows);
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->done, 1);
    tc::mbar_init(&bars->rows_ready[0], kBtRows);
    tc::mbar_init(&bars->rows_ready[1], kBtRows);
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  char* sK = smem + L::kK;
  char* sV = smem + L::kV;
  char* sStage = smem + L::kStage;

  if (warp == 1) {
    // the whole warp runs the issuer loop; elect.sync picks the issuing lane
    bt_kv_mma<D>(bars, tmem, tc::smem_addr(sK), tc::smem_addr(sV), tc::smem_addr(sStage), n_rt,
                 abort_flag);
  } else if (warp == 0) {
    // ---------------------------------------------------------- producer
    const int ent = bt_entry(lst, jt * kBtGroupsPerTile + (lane & 15), a.group);
    const int64_t head_group0 = (int64_t)h * (a.t_cap / a.group);
    const int zero_group = (int)((int64_t)a.Hkv * (a.t_cap / a.group));
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_q);
      tc::tma_prefetch_desc(&tm_do);
      tc::mbar_arrive_expect_tx(&bars->kv_full, 2 * kBtGroupsPerTile * L::kHalves * 1024);
    }
    __syncwarp();
    bt_load_tile<D>(sK, &tm_k1, &tm_k8, ent, head_group0, zero_group, &bars->kv_full, lane);
    bt_load_tile<D>(sV, &tm_v1, &tm_v8, ent, head_group0, zero_group, &bars->kv_full, lane);
    const int pos0 = (int)(b0 - a.q_start);
    int issued = 0;
    for (int rt = 0; rt < n_rt; ++rt) {
      const int s = rt & 1;
      int ok = 1;
      if (rt >= 2 && lane == 0)
        ok = tc::mbar_wait(&bars->stage_empty[s], ((rt - 2) >> 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0)
        tc::mbar_arrive_expect_tx(&bars->stage_full[s], 2 * L::kRowTileBytes);
      __syncwarp();
      if (lane < 2 * L::kHalves) {
        const int which = lane / L::kHalves, hf = lane % L::kHalves;   // 0: Q, 1: dO
        tc::tma_load_3d(sStage + (s * 2 + which) * L::kRowTileBytes + hf * L::kHalfBytes,
                        which ? &tm_do : &tm_q, hf * 64, h * a.G,
                        pos0 + rt * (kBtRows / a.G), &bars->stage_full[s]);
      }
      issued = rt + 1;
    }
    // no copy may still be landing when the CTA leaves
    if (lane == 0) {
      const uint64_t t0 = tc::globaltimer_ns();
      while (!tc::mbar_try_wait(&bars->kv_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
      }
      for (int rt = max(0, issued - 2); rt < issued; ++rt) {
        const uint64_t t1 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&bars->stage_full[rt & 1], (rt >> 1) & 1) &&
               tc::globaltimer_ns() - t1 < tc::kWaitLimitNs) {
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- P, dS
    // thread r = token r of the tile (TMEM lane r): S^T and dP^T rows hold the
    // token's scores against the 128 rows of the current row tile
    const int r = tid - 128;
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off, t_dp = tmem + lane_off + 128;
    const int ent = bt_entry(lst, jt * kBtGroupsPerTile + (r >> 3), a.group);
    const int64_t tok = (int64_t)ent * a.group + (r & 7);
    const bool tok_ok = ent >= 0 && tok < T;
    // the token is attended by rows whose position is >= tok, i.e. unit rows
    // >= G * (tok - b0)
    const int64_t first_row = (int64_t)a.G * (tok - b0);
    bool ok = true;
    for (int rt = 0; rt < n_rt; ++rt) {
      float* lse_s = rowvals + (rt & 1) * 2 * kBtRows;
      float* d_s = lse_s + kBtRows;
      {
        const int ur = rt * kBtRows + r;
        const bool live = ur < nrows;
        const int64_t row = (b0 - a.q_start + (live ? ur / a.G : 0)) * a.Hq + (int64_t)h * a.G +
                            (live ? ur % a.G : 0);
        lse_s[r] = live ? w.lse[row] * kLog2e : INFINITY;   // dead rows: p = 0
        d_s[r] = live ? w.d_q[row * D] : 0.f;
      }
      // every thread reads all 128 values: wait until they are written (the
      // buffer of row tile rt - 2 was last read before p_full of rt - 2,
      // which the MMA awaited before S^T of rt - 1 completed)
      tc::mbar_arrive(&bars->rows_ready[rt & 1]);
      if (!(ok = tc::mbar_wait_warp(&bars->rows_ready[rt & 1], (rt >> 1) & 1, abort_flag))) break;
      if (!(ok = tc::mbar_wait_warp(&bars->sdp_full, rt & 1, abort_flag))) break;
      tc::fence_after_sync();
      const int64_t cmin = first_row - (int64_t)rt * kBtRows;   // columns below are masked
#pragma unroll
      for (int qq = 0; qq < kBtRows / 32; ++qq) {
        uint32_t sr[32], dr[32];
        tc::tmem_ld32(t_s + qq * 32, sr);
        tc::tmem_ld32(t_dp + qq * 32, dr);
        tc::tmem_wait_ld();
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int col = qq * 32 + c;
          const float2 l2 = *reinterpret_cast<const float2*>(lse_s + col);
          const float2 D2 = *reinterpret_cast<const float2*>(d_s + col);
          const bool v0 = tok_ok && col >= cmin, v1 = tok_ok && col + 1 >= cmin;
          const float p0 = v0 ? tc::ex2(fmaf(__uint_as_float(sr[c]), w.scale_log2, -l2.x)) : 0.f;
          const float p1 = v1 ? tc::ex2(fmaf(__uint_as_float(sr[c + 1]), w.scale_log2, -l2.y)) : 0.f;
          const float ds0 = v0 ? p0 * (__uint_as_float(dr[c]) - D2.x) : 0.f;
          const float ds1 = v1 ? p1 * (__uint_as_float(dr[c + 1]) - D2.y) : 0.f;
          pp[c >> 1] = tc::pack_bf162(p0, p1);
          dd[c >> 1] = tc::pack_bf162(ds0, ds1);
        }
        tc::tmem_st16(t_s + qq * 16, pp);     // P^T over the columns of S^T already read
        tc::tmem_st16(t_dp + qq * 16, dd);    // dS^T likewise
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full);
    }
    // ---- flush: dV, dK (scaled) of this token into the global sums
    if (ok && tc::mbar_wait_warp(&bars->acc_full, 0, abort_flag)) {
      tc::fence_after_sync();
      float* dv = w.d_v + ((int64_t)h * a.t_cap + (tok_ok ? tok : 0)) * D;
      float* dk = w.d_k + ((int64_t)h * a.t_cap + (tok_ok ? tok : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t vr[32], kr[32];
        tc::tmem_ld32(tmem + lane_off + 256 + c * 32, vr);
        tc::tmem_ld32(tmem + lane_off + 384 + c * 32, kr);
        tc::tmem_wait_ld();
        if (tok_ok) {
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            atomicAdd(reinterpret_cast<float4*>(dv + c * 32 + x),
                      make_float4(__uint_as_float(vr[x]), __uint_as_float(vr[x + 1]),
                                  __uint_as_float(vr[x + 2]), __uint_as_float(vr[x + 3])));
            atomicAdd(reinterpret_cast<float4*>(dk + c * 32 + x),
                      make_float4(__uint_as_float(kr[x]) * w.scale,
                                  __uint_as_float(kr[x + 1]) * w.scale,
                                  __uint_as_float(kr[x + 2]) * w.scale,
                                  __uint_as_float(kr[x + 3]) * w.scale));
          }
        }
      }
    }
  }

  griddep_launch();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ

template <int D>
struct BtQLayout {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kBtRows * 128;
  static constexpr int kRowTileBytes = kHalves * kHalfBytes;
  static constexpr int kGroupBytes = kHalves * 8 * 128;
  static constexpr int kSlotBytes = kBtGroupsPerTile * kGroupBytes;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kRowTileBytes;
  static constexpr int kSlot = kDO + kRowTileBytes;
  static constexpr int kBar = kSlot + kTcSlots * kSlotBytes;
  static constexpr int kList = kBar + 256;
  static constexpr size_t smem_bytes(int max_list) {
    return 1024 + (size_t)kList + (size_t)max_list * 4;
  }
};

struct BtQBars {
  uint64_t q_full, full[kTcSlots], empty[kTcSlots], sdp_full, p_full, dq_full, done;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__device__ __noinline__ void bt_q_mma(BtQBars* bars, uint32_t tmem, uint32_t q_base,
                                     uint32_t do_base, uint32_t slot_base, int n_tiles,
                                     volatile int* abort_flag) {
  using L = BtQLayout<D>;
  constexpr uint32_t kIdS = tc::idesc_f16(kBtRows, kBtTok, 1, 0);   // M rows, N tokens
  constexpr uint32_t kIdQ = tc::idesc_f16(kBtRows, D, 1, 1);        // M rows, N = d (MN-major B)
  const uint64_t q_desc = tc::sdesc_sw128(q_base, 16, 1024);
  const uint64_t do_desc = tc::sdesc_sw128(do_base, 16, 1024);
  const uint64_t kv_kmaj0 = tc::sdesc_sw128(slot_base, 16, L::kGroupBytes);
  const uint64_t k_mn0 = tc::sdesc_sw128(slot_base, 1024, L::kGroupBytes);
  bool ok = tc::mbar_wait_warp(&bars->q_full, 0, abort_flag);
  for (int j = 0; ok && j < n_tiles; ++j) {
    const int nk = 2 * j, sk = nk % kTcSlots, nv = nk + 1, sv = nv % kTcSlots;
    if (!(ok = tc::mbar_wait_warp(&bars->full[sk], (nk / kTcSlots) & 1, abort_flag))) break;
    tc::fence_after_sync();
    const uint64_t kd = kv_kmaj0 + (uint64_t)((sk * L::kSlotBytes) >> 4);
    const uint64_t vd = kv_kmaj0 + (uint64_t)((sv * L::kSlotBytes) >> 4);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t ko = (uint32_t)(((k >> 2) * 1024 + (k & 3) * 32) >> 4);
      const uint32_t qo = (uint32_t)(((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4);
      tc::mma_ss_warp(tmem + 0, q_desc + qo, kd + ko, kIdS, k > 0);            // S = Q K^T
    }
    if (!(ok = tc::mbar_wait_warp(&bars->full[sv], (nv / kTcSlots) & 1, abort_flag))) break;
    tc::fence_after_sync();
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t ko = (uint32_t)(((k >> 2) * 1024 + (k & 3) * 32) >> 4);
      const uint32_t qo = (uint32_t)(((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4);
      tc::mma_ss_warp(tmem + 128, do_desc + qo, vd + ko, kIdS, k > 0);         // dP = dO V^T
    }
    tc::mma_commit_warp(&bars->sdp_full);
    if (!(ok = tc::mbar_wait_warp(&bars->p_full, j & 1, abort_flag))) break;
    tc::fence_after_sync();
    const uint64_t kmn = k_mn0 + (uint64_t)((sk * L::kSlotBytes) >> 4);
#pragma unroll
    for (int k = 0; k < kBtTok / 16; ++k)
      tc::mma_ts_warp(tmem + 256, tmem + 0 + k * 8,
                      kmn + (uint64_t)((2 * k * L::kGroupBytes) >> 4), kIdQ,
                      (j > 0 || k > 0) ? 1u : 0u);                         // dQ += dS K
    tc::mma_commit_warp(&bars->empty[sk]);
    tc::mma_commit_warp(&bars->empty[sv]);
  }
  tc::mma_commit_warp(&bars->dq_full);
  tc::mma_commit_warp(&bars->done);
  const uint64_t t0 = tc::globaltimer_ns();
  while (!tc::mbar_try_wait(&bars->done, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
  }
}

template <int D>
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k1,
                  const __grid_constant__ CUtensorMap tm_k8,
                  const __grid_constant__ CUtensorMap tm_v1,
                  const __grid_constant__ CUtensorMap tm_v8, BtArgs w) {
  using L = BtQLayout<D>;
  const AttendArgs& a = w.a;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BtQBars* bars = reinterpret_cast<BtQBars*>(smem + L::kBar);
  int* list = reinterpret_cast<int*>(smem + L::kList);
  volatile int* abort_flag = &bars->abort;

  griddep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y, h = blockIdx.z;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  const int row0 = blockIdx.x * kBtRows;
  if (row0 >= nrows) return;

  if (tid == 0) {
    bars->abort = 0;
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kTcSlots; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    tc::mbar_init(&bars->sdp_full, 1);
    tc::mbar_init(&bars->p_full, kBtRows);
    tc::mbar_init(&bars->dq_full, 1);
    tc::mbar_init(&bars->done, 1);
    tc::fence_mbar_init();
  }
  __shared__ int s_inv;
  if (tid == 0) s_inv = 0;
  __syncthreads();
  char* sQ = smem + L::kQ;
  char* sDO = smem + L::kDO;
  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_q);
      tc::tma_prefetch_desc(&tm_do);
      tc::mbar_arrive_expect_tx(&bars->q_full, 2 * L::kRowTileBytes);
    }
    __syncwarp();
    if (lane < 2 * L::kHalves) {
      const int which = lane / L::kHalves, hf = lane % L::kHalves;
      tc::tma_load_3d((which ? sDO : sQ) + hf * L::kHalfBytes, which ? &tm_do : &tm_q, hf * 64,
                      h * a.G, (int)(b0 - a.q_start) + row0 / a.G, &bars->q_full);
    }
  }
  int n_nondiag;
  bool inv = false;
  const int n_list = build_group_list_tc(a, b, h, b0, T, list, &n_nondiag, &inv);
  if (inv) s_inv = 1;
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const bool any_invalid = s_inv != 0;
  const int n_tiles = (n_list + kBtGroupsPerTile - 1) / kBtGroupsPerTile;
  auto slot_ptr = [&](int s) { return smem + L::kSlot + s * L::kSlotBytes; };

  if (warp == 1) {
    // the whole warp runs the issuer loop; elect.sync picks the issuing lane
    bt_q_mma<D>(bars, tmem, tc::smem_addr(sQ), tc::smem_addr(sDO), tc::smem_addr(slot_ptr(0)),
                n_tiles, abort_flag);
  } else if (warp == 0) {
    // ---------------------------------------------------------- producer
    // ring load n: K of tile n/2 (n even) or V (n odd), into slot n % 4
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k1);
      tc::tma_prefetch_desc(&tm_k8);
      tc::tma_prefetch_desc(&tm_v1);
      tc::tma_prefetch_desc(&tm_v8);
    }
    const int64_t head_group0 = (int64_t)h * (a.t_cap / a.group);
    const int zero_group = (int)((int64_t)a.Hkv * (a.t_cap / a.group));
    int last_use[kTcSlots];
#pragma unroll
    for (int s = 0; s < kTcSlots; ++s) last_use[s] = -1;
    for (int n = 0; n < 2 * n_tiles; ++n) {
      const int s = n % kTcSlots, u = n / kTcSlots, j = n >> 1;
      int ok = 1;
      if (n >= kTcSlots && lane == 0) ok = tc::mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int li = j * kBtGroupsPerTile + (lane & 15);
      const int ent = li < n_list ? list[li] : -1;
      if (lane == 0)
        tc::mbar_arrive_expect_tx(&bars->full[s], kBtGroupsPerTile * L::kHalves * 1024);
      __syncwarp();
      bt_load_tile<D>(slot_ptr(s), (n & 1) ? &tm_v1 : &tm_k1, (n & 1) ? &tm_v8 : &tm_k8, ent,
                      head_group0, zero_group, &bars->full[s], lane);
      last_use[s] = u;
    }
    if (lane == 0) {
      for (int s = 0; s < kTcSlots; ++s) {
        if (last_use[s] < 0) continue;
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&bars->full[s], last_use[s] & 1) &&
               tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- dS
    const int r = tid - 128;                   // row within the tile (TMEM lane)
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off, t_dp = tmem + lane_off + 128;
    const int ur = row0 + r;
    const bool live = ur < nrows;
    const int64_t pos = b0 + (live ? ur / a.G : 0);
    const int64_t row = (pos - a.q_start) * a.Hq + (int64_t)h * a.G + (live ? ur % a.G : 0);
    const float lse_l2 = live ? w.lse[row] * kLog2e : INFINITY;   // dead rows: p = 0
    const float Dr = live ? w.d_q[row * D] : 0.f;                  // before d_q is written
    const int pos32 = (int)pos;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!(ok = tc::mbar_wait_warp(&bars->sdp_full, j & 1, abort_flag))) break;
      tc::fence_after_sync();
      const bool need_mask = any_invalid || (j * kBtGroupsPerTile + kBtGroupsPerTile > n_nondiag);
#pragma unroll
      for (int qq = 0; qq < kBtTok / 32; ++qq) {
        uint32_t sr[32], dr[32];
        tc::tmem_ld32(t_s + qq * 32, sr);
        tc::tmem_ld32(t_dp + qq * 32, dr);
        tc::tmem_wait_ld();
        int lim[4];                            // valid columns c <= lim of each group
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          lim[g4] = 7;
          if (need_mask) {
            const int li = j * kBtGroupsPerTile + qq * 4 + g4;
            const int ent = li < n_list ? list[li] : -1;
            lim[g4] = ent < 0 ? -1 : pos32 - ent * a.group;
          }
        }
        if (!live) {
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) lim[g4] = -1;
        }
        uint32_t dd[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int l = lim[c >> 3];
          const bool v0 = (c & 7) <= l, v1 = ((c + 1) & 7) <= l;
          const float p0 = v0 ? tc::ex2(fmaf(__uint_as_float(sr[c]), w.scale_log2, -lse_l2)) : 0.f;
          const float p1 = v1 ? tc::ex2(fmaf(__uint_as_float(sr[c + 1]), w.scale_log2, -lse_l2)) : 0.f;
          const float ds0 = v0 ? p0 * (__uint_as_float(dr[c]) - Dr) : 0.f;
          const float ds1 = v1 ? p1 * (__uint_as_float(dr[c + 1]) - Dr) : 0.f;
          dd[c >> 1] = tc::pack_bf162(ds0, ds1);
        }
        tc::tmem_st16(t_s + qq * 16, dd);      // dS over the columns of S already read
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full);
    }
    // ---- dQ of this row, scaled, stored once
    if (ok && tc::mbar_wait_warp(&bars->dq_full, 0, abort_flag)) {
      tc::fence_after_sync();
      float* dst = w.d_q + row * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t qr[32];
        tc::tmem_ld32(tmem + lane_off + 256 + c * 32, qr);
        tc::tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dst + c * 32 + x) =
                make_float4(__uint_as_float(qr[x]) * w.scale, __uint_as_float(qr[x + 1]) * w.scale,
                            __uint_as_float(qr[x + 2]) * w.scale,
                            __uint_as_float(qr[x + 3]) * w.scale);
        }
      }
    }
  }

  griddep_launch();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace hga
