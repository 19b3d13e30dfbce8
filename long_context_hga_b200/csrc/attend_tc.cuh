// Step 4 on the sm_100a tensor cores: gathered exact-token attention with
// tcgen05.mma, TMEM accumulators and TMA gathers of the routed groups.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: exact token K/V
// of the kept groups plus the sink and local windows feed softmax attention.
//
// One CTA = 256 query rows of one (query block, KV head) unit, as two 128-row
// tiles Q0/Q1 (rows are (position, query head) pairs, so the G heads that
// share the KV head reuse every gathered K/V tile).  K/V arrive in 128-token
// tiles (16 routed 8-token groups); each group is one contiguous 8 x d span of
// the head-major cache and is fetched by TMA as 8-row x 128-byte boxes with
// the 128-byte swizzle, which is exactly one swizzle atom of the tcgen05
// operand layout, so arbitrary group lists need no repacking.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q first (before the group list is known), then
//               K/V tiles into a 4-slot ring (one K or V tile per slot)
//   warp 1      TMEM owner and MMA issuer (the warp runs the loop, one
//               elected lane issues):
//                 S_i = Q_i K^T   (bf16 x bf16 -> fp32, K-major A and B)
//                 O_i += P_i V    (fp16 P from TMEM x fp16 V, MN-major B)
//   warps 2-3   convert each V tile bf16 -> fp16 in place (exact below 65504;
//               P kept in fp16 has 11 significant bits) and zero rows that
//               hold no attended token; with V stored as fp16 (VF16) only
//               the zeroing remains
//   warps 4-7   softmax of tile Q0, warps 8-11 softmax of tile Q1: one thread
//               per row reads its S row from TMEM, applies the causal / padding
//               mask, keeps the running max and sum in fp32, writes P (fp16)
//               over its S columns and rescales O only when the max grows by
//               more than 2^8 (exact: O and the sum always share one max)
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
// While one softmax warpgroup works, the MMA warp runs the other tile's
// products, so the tensor pipe and the exponentials overlap.
#pragma once
#include "attend.cuh"
#include "tc.cuh"

namespace hga {

constexpr int kTcRows = 128;              // rows per Q tile (MMA M)
constexpr int kTcTok = 128;               // tokens per K/V tile (MMA N of S)
constexpr int kTcGroupsPerTile = kTcTok / 8;
constexpr int kTcThreads = 384;
constexpr int kTcSlots = 4;               // K/V ring: one K or V tile per slot
constexpr int kTcMaxList = 4608;          // group-list slots in shared memory
constexpr float kTcRescaleLog2 = 8.0f;

struct TcArgs {
  AttendArgs a;
  int rows_per_cta;                       // 256
  int64_t stall_load;                     // test hook: the producer stops before this
                                          // load of the ring (-1: never)
};

template <int D>
struct TcLayout {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kTcRows * 128;                 // 16 KB
  static constexpr int kQBytes = 2 * kHalves * kHalfBytes;         // 2 tiles
  static constexpr int kGroupBytes = kHalves * 8 * 128;            // one 8-token group
  static constexpr int kSlotBytes = kTcGroupsPerTile * kGroupBytes;  // one K or V tile
  static constexpr int kQOff = 0;
  static constexpr int kSlotOff = kQOff + kQBytes;
  static constexpr int kBarOff = kSlotOff + kTcSlots * kSlotBytes;
  static constexpr int kListOff = kBarOff + 512;
  static constexpr size_t smem_bytes(int max_list) {
    return 1024 + (size_t)kListOff + (size_t)max_list * 4;
  }
};

struct TcBars {
  uint64_t q_full, full[kTcSlots], empty[kTcSlots], v_ready[kTcSlots];
  uint64_t s_full[2], p_full[2], o_full[2], done;
  uint64_t ostage[2];    // per Q tile: all rows of O staged in shared memory
  uint32_t tmem_base;
  int abort;
};


// The unit's group list (sink, routed, local window, diagonal; see
// build_group_list) built by the whole CTA with one round of global reads:
// every thread reads the routed entries its list slots would hold (and the
// ones before them, for the ascending check) in the same round as the routed
// count, instead of after it.  Invalid routed entries become -1 and are
// reported; a list longer than the shared buffer gives 0 entries (reported).
__device__ __forceinline__ int build_group_list_tc(const AttendArgs& a, int b, int h, int64_t b0,
                                                   int64_t T, int* list, int* n_nondiag,
                                                   bool* any_invalid) {
  const int g = a.group;
  const int64_t sink_end = min((int64_t)a.sink, b0);
  const int n_s = (int)(sink_end / g);
  const int32_t* routed = a.group_idx + ((int64_t)h * a.n_blocks + b) * a.cap_g;
  const int64_t loc_lo = max(sink_end, b0 - a.local);
  const int n_l = (int)((b0 - loc_lo) / g);
  const int64_t b_end = min(b0 + a.qblock, T);
  const int n_d = (int)((b_end - b0 + g - 1) / g);
  const int n_max = (int)min((int64_t)a.max_list, (int64_t)n_s + a.cap_g + n_l + n_d);
  int n_r = a.group_cnt[(int64_t)h * a.n_blocks + b];
  const int64_t lo_tok = a.sink, hi_tok = b0 - a.local;
  bool bad = false;
  for (int i = threadIdx.x; i < n_max; i += blockDim.x) {
    const int r = i - n_s;
    const int cur = (r >= 0 && r < a.cap_g) ? routed[r] : -1;
    const int prev = (r >= 1 && r <= a.cap_g) ? routed[r - 1] : -1;
    int nr = n_r;
    if (nr < 0 || nr > a.cap_g) nr = 0;
    int e;
    if (i < n_s) e = i;
    else if (i < n_s + nr) {
      e = cur;
      const bool ok = (int64_t)e * g >= lo_tok && ((int64_t)e + 1) * g <= hi_tok &&
                      (r == 0 || e > prev);
      if (!ok) { e = -1; bad = true; }
    } else if (i < n_s + nr + n_l) e = (int)(loc_lo / g) + (i - n_s - nr);
    else if (i < n_s + nr + n_l + n_d) e = (int)(b0 / g) + (i - n_s - nr - n_l);
    else continue;
    list[i] = e;
  }
  if (n_r < 0 || n_r > a.cap_g) { bad = true; n_r = 0; }
  if (bad) { report(HGA_ERR_DEVICE_CHECK); *any_invalid = true; }
  const int n = n_s + n_r + n_l + n_d;
  *n_nondiag = n_s + n_r + n_l;
  if (n > a.max_list) {
    if (threadIdx.x == 0) report(HGA_ERR_DEVICE_CHECK);
    return 0;
  }
  return n;
}

// The MMA issuer.  Per tile j it issues, for each Q tile i, O_i += P_i(j-1)
// V(j-1) (once softmax has written P_i(j-1)) and then S_i(j) = Q_i K(j)^T; a
// last round issues the final P.V.  The whole warp runs the loop (waits
// included) and elect.sync picks the lane that issues each product and
// commit: with the loop's values warp-uniform the products issue faster than
// from a loop run by one lane inside a divergent branch (the attention step
// measured 65.5 -> 61.5 us).  It is kept out of line so that its loop runs
// from registers of its own (inlined into the kernel, whose softmax code sets
// the register allocation, the loop reloaded spilled values per MMA).
template <int D>
__device__ __noinline__ void tc_mma_issuer(TcBars* bars, uint32_t tmem, uint32_t q_base,
                                          uint32_t slot_base, int nq, int n_tiles,
                                          volatile int* abort_flag) {
  using L = TcLayout<D>;
  constexpr uint32_t kIdS = tc::idesc_f16(kTcRows, kTcTok, 1, 0);
  constexpr uint32_t kIdPV = tc::idesc_f16(kTcRows, D, 0, 1);
  bool ok = tc::mbar_wait_warp(&bars->q_full, 0, abort_flag);
  tc::fence_after_sync();
  const uint64_t q_desc0 = tc::sdesc_sw128(q_base, 16, 1024);
  const uint64_t k_desc0 = tc::sdesc_sw128(slot_base, 16, L::kGroupBytes);
  const uint64_t v_desc0 = tc::sdesc_sw128(slot_base, 1024, L::kGroupBytes);
  for (int j = 0; ok && j <= n_tiles; ++j) {
    const bool has_s = j < n_tiles, has_pv = j > 0;
    const int nk = 2 * j, sk = nk % kTcSlots;
    const int nv = 2 * j - 1, sv = (nv + kTcSlots) % kTcSlots;
    if (has_pv &&
        !(ok = tc::mbar_wait_warp(&bars->v_ready[sv], (nv / kTcSlots) & 1, abort_flag)))
      break;
    const uint64_t kd = k_desc0 + (uint64_t)((sk * L::kSlotBytes) >> 4);
    const uint64_t vd = v_desc0 + (uint64_t)((sv * L::kSlotBytes) >> 4);
    for (int i = 0; i < nq; ++i) {
      if (has_pv) {
        if (!(ok = tc::mbar_wait_warp(&bars->p_full[i], (j - 1) & 1, abort_flag))) break;
        tc::fence_after_sync();
        const uint32_t acc0 = j == 1 ? 0u : 1u;
        const uint32_t d_o = tmem + 256 + i * 128, a_p = tmem + i * 128;
#pragma unroll
        for (int k = 0; k < kTcTok / 16; ++k)
          tc::mma_ts_warp(d_o, a_p + k * 8, vd + (uint64_t)((2 * k * L::kGroupBytes) >> 4), kIdPV,
                          k > 0 ? 1u : acc0);
        tc::mma_commit_warp(&bars->o_full[i]);
      }
      if (has_s) {
        if (i == 0) {
          if (!(ok = tc::mbar_wait_warp(&bars->full[sk], (nk / kTcSlots) & 1, abort_flag))) break;
          tc::fence_after_sync();
        }
        const uint64_t qd = q_desc0 + (uint64_t)((i * L::kHalves * L::kHalfBytes) >> 4);
        const uint32_t d_s = tmem + i * 128;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_ss_warp(d_s, qd + (uint64_t)((((k >> 2) * L::kHalfBytes) + (k & 3) * 32) >> 4),
                          kd + (uint64_t)((((k >> 2) * 1024) + (k & 3) * 32) >> 4), kIdS, k > 0);
        tc::mma_commit_warp(&bars->s_full[i]);
      }
    }
    if (!ok) break;
    if (has_pv) tc::mma_commit_warp(&bars->empty[sv]);
    if (has_s) tc::mma_commit_warp(&bars->empty[sk]);
  }
  // drain: every MMA issued so far has completed before TMEM is freed
  tc::mma_commit_warp(&bars->done);
  const uint64_t t0 = tc::globaltimer_ns();
  while (!tc::mbar_try_wait(&bars->done, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
  }
}

template <int D, bool VF16 = false>
__global__ void __launch_bounds__(kTcThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k1,
                     const __grid_constant__ CUtensorMap tm_k8,
                     const __grid_constant__ CUtensorMap tm_v1,
                     const __grid_constant__ CUtensorMap tm_v8,
                     const __grid_constant__ CUtensorMap tm_o, TcArgs args) {
  using L = TcLayout<D>;
  const AttendArgs& a = args.a;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(smem + L::kBarOff);
  int* list = reinterpret_cast<int*>(smem + L::kListOff);
  volatile int* abort_flag = &bars->abort;

  // Every input is read after waiting for the previous kernel, except Q with
  // q_early (complete before that kernel can let this one start): its load
  // is then requested first and overlaps that kernel's tail.
  if (!a.q_early) griddep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y, h = blockIdx.z;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  // first unit row of this CTA; rows of positions before pos_lo are skipped
  const int skip = (int)min((int64_t)npos, max((int64_t)0, a.pos_lo - b0)) * a.G;
  const int row0 = skip + blockIdx.x * args.rows_per_cta;
  if (row0 >= nrows) return;
  const int nq = (nrows - row0) > kTcRows ? 2 : 1;     // Q tiles with live rows

  // ---- prologue: barriers, the Q load, group list, TMEM.  Q depends on
  // the unit only, so it is requested before the group list is read.
  if (tid == 0) {
    bars->abort = 0;
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kTcSlots; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
      tc::mbar_init(&bars->v_ready[s], 64);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars->s_full[i], 1);
      tc::mbar_init(&bars->p_full[i], kTcRows);
      tc::mbar_init(&bars->o_full[i], 1);
    }
    tc::mbar_init(&bars->done, 1);
    tc::mbar_init(&bars->ostage[0], kTcRows);
    tc::mbar_init(&bars->ostage[1], kTcRows);
    tc::fence_mbar_init();
  }
  __shared__ int s_inv;
  if (tid == 0) s_inv = 0;
  __syncthreads();
  char* sQ = smem + L::kQOff;
  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_q);
      tc::mbar_arrive_expect_tx(&bars->q_full, nq * L::kHalves * L::kHalfBytes);
    }
    __syncwarp();
    if (lane < nq * L::kHalves) {
      const int i = lane / L::kHalves, hf = lane % L::kHalves;
      const int pos0 = (int)(b0 - a.q_start) + row0 / a.G;
      tc::tma_load_3d(sQ + (i * L::kHalves + hf) * L::kHalfBytes, &tm_q, hf * 64, h * a.G,
                      pos0 + i * (kTcRows / a.G), &bars->q_full);
    }
  }
  if (a.q_early) griddep_wait();
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
  const int n_tiles = (n_list + kTcGroupsPerTile - 1) / kTcGroupsPerTile;
  const int n_loads = 2 * n_tiles;             // K0 V0 K1 V1 ... through the ring

  auto slot_ptr = [&](int s, int half) {
    return smem + L::kSlotOff + s * L::kSlotBytes + half * 1024;
  };

  if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    tc_mma_issuer<D>(bars, tmem, tc::smem_addr(sQ), tc::smem_addr(slot_ptr(0, 0)), nq, n_tiles,
                     abort_flag);
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Load n of the ring is K_{n/2} (n even) or V_{n/2} (n odd), into slot
    // n % kTcSlots.  A slot holds 16 groups as [group][half][8 rows][128 B]
    // (2 KB per group, 128-byte swizzle), which is what one box of the 4-D
    // tensor view (64 dims, 8 rows, 2 halves, group) lands as; 8 aligned
    // consecutive groups (sink, local window, diagonal, adjacent routed
    // groups) come in one 16 KB box.  Lane e < 16 owns entry e of the tile.
    // (Q was requested in the prologue)
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k1);
      tc::tma_prefetch_desc(&tm_k8);
      tc::tma_prefetch_desc(&tm_v1);
      tc::tma_prefetch_desc(&tm_v8);
    }
    int last_use[kTcSlots];
#pragma unroll
    for (int s = 0; s < kTcSlots; ++s) last_use[s] = -1;
    const int e = lane & 15;
    const int64_t head_group0 = (int64_t)h * (a.t_cap / a.group);
    for (int n = 0; n < n_loads; ++n) {
      const int s = n % kTcSlots, u = n / kTcSlots, j = n >> 1;
      if (n == args.stall_load) break;      // test hook: this load is never issued
      int ok = 1;
      if (n >= kTcSlots && lane == 0) ok = tc::mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int li = j * kTcGroupsPerTile + e;
      const int ent = li < n_list ? list[li] : -1;
      // runs: entries 8r..8r+7 are 8 consecutive valid groups
      const int ent0 = __shfl_sync(0xffffffffu, ent, e & ~7);
      const bool consec = ent >= 0 && ent0 >= 0 && ent == ent0 + (e & 7);
      const unsigned cons_mask = __ballot_sync(0xffffffffu, lane < 16 && consec);
      const bool run = ((cons_mask >> (e & ~7)) & 0xffu) == 0xffu;
      const unsigned valid = __ballot_sync(0xffffffffu, lane < 16 && ent >= 0);
      if (lane == 0)
        tc::mbar_arrive_expect_tx(&bars->full[s], __popc(valid) * L::kHalves * 1024);
      __syncwarp();
      if (lane < 16 && ent >= 0) {
        const bool vt = n & 1;
        const int gcoord = (int)(head_group0 + ent);
        if (run) {
          if ((e & 7) == 0)
            tc::tma_load_4d(slot_ptr(s, 0) + e * L::kGroupBytes, vt ? &tm_v8 : &tm_k8, 0, 0, 0,
                            gcoord, &bars->full[s]);
        } else {
          tc::tma_load_4d(slot_ptr(s, 0) + e * L::kGroupBytes, vt ? &tm_v1 : &tm_k1, 0, 0, 0,
                          gcoord, &bars->full[s]);
        }
      }
      last_use[s] = u;
    }
    // make sure no copy is still landing in shared memory when we leave
    if (lane == 0) {
      for (int s = 0; s < kTcSlots; ++s) {
        if (last_use[s] < 0) continue;
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&bars->full[s], last_use[s] & 1) &&
               tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ V converter
    // bf16 -> fp16 in place (exact below 65504; a larger magnitude becomes
    // inf and is caught by the epilogue's finite check), then rows that hold
    // no attended token (padding entries, tokens past the context) are
    // zeroed so that P = 0 always meets finite V.
    const int ct = tid - 64;   // 0..63
    constexpr int kChunks = L::kSlotBytes / 16;
    auto cvt4 = [](uint4& r) {
      uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        w[t] = tc::pack_half2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xffff0000u));
    };
    for (int j = 0; j < n_tiles; ++j) {
      const int nv = 2 * j + 1, s = nv % kTcSlots;
      if (!tc::mbar_wait_warp(&bars->full[s], (nv / kTcSlots) & 1, abort_flag)) break;
      const int li0 = j * kTcGroupsPerTile;
      bool clean = li0 + kTcGroupsPerTile <= n_list && !any_invalid;
      if (clean) clean = ((int64_t)list[li0 + kTcGroupsPerTile - 1] + 1) * a.group <= T;
      char* base = slot_ptr(s, 0);
      if (VF16 && clean) {
        // fp16 V as loaded; nothing to do
      } else if (clean) {
#pragma unroll
        for (int q0 = 0; q0 < kChunks; q0 += 64 * 8) {
          uint4 raw[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) raw[x] = *reinterpret_cast<const uint4*>(base + (q0 + x * 64 + ct) * 16);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            cvt4(raw[x]);
            *reinterpret_cast<uint4*>(base + (q0 + x * 64 + ct) * 16) = raw[x];
          }
        }
      } else {
        for (int q = ct; q < kChunks; q += 64) {
          // offset -> (group, row): [group][half][8 rows][128 B]; rows that
          // were not loaded hold stale bytes and are only zeroed
          const int g = (q * 16) / L::kGroupBytes;
          const int rr = ((q * 16) % 1024) / 128;
          const int li = li0 + g;
          const int ent = li < n_list ? list[li] : -1;
          const bool live = ent >= 0 && (int64_t)ent * a.group + rr < T;
          if constexpr (VF16) {
            if (!live) *reinterpret_cast<uint4*>(base + q * 16) = make_uint4(0, 0, 0, 0);
          } else {
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (live) {
              raw = *reinterpret_cast<const uint4*>(base + q * 16);
              cvt4(raw);
            }
            *reinterpret_cast<uint4*>(base + q * 16) = raw;
          }
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars->v_ready[s]);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int i = (warp - 4) >> 2;              // Q tile of this warpgroup
    const int quarter = warp & 3;               // TMEM lane quarter
    const int r = quarter * 32 + lane;          // row within the Q tile
    const int unit_row = row0 + i * kTcRows + r;
    const bool row_live = (i < nq) && unit_row < nrows;
    const int64_t pos = b0 + (row_live ? unit_row / a.G : 0);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + i * 128;
    const uint32_t t_o = tmem + lane_off + 256 + i * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = i < nq;
    for (int j = 0; ok && j < n_tiles; ++j) {
      if (!(ok = tc::mbar_wait_warp(&bars->s_full[i], j & 1, abort_flag))) break;
      tc::fence_after_sync();
      // The whole S row (128 columns) is read from TMEM once, masked,
      // reduced to its max, then turned into P in place.
      const bool need_mask = any_invalid || (j * kTcGroupsPerTile + kTcGroupsPerTile > n_nondiag);
      uint32_t sr[kTcTok];
#pragma unroll
      for (int c = 0; c < kTcTok / 32; ++c) tc::tmem_ld32(t_s + c * 32, sr + c * 32);
      tc::tmem_wait_ld();
      if (need_mask) {
        // token indices fit in 32 bits on this path (Hkv * t_cap < 2^31)
        const int pos32 = (int)pos;
#pragma unroll
        for (int e = 0; e < kTcGroupsPerTile; ++e) {
          const int li = j * kTcGroupsPerTile + e;
          const int ent = li < n_list ? list[li] : -1;
          const int lim = ent < 0 ? -1 : pos32 - ent * 8;   // valid columns c <= lim
#pragma unroll
          for (int c = 0; c < 8; ++c)
            if (c > lim) sr[e * 8 + c] = __float_as_uint(-INFINITY);
        }
      }
      // 8 independent partial maxima (no 128-long dependency chain), two
      // new columns per three-input max
      float mx8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) mx8[x] = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTcTok; c += 2)
        mx8[(c >> 1) & 7] = tc::fmax3(mx8[(c >> 1) & 7], __uint_as_float(sr[c]),
                                      __uint_as_float(sr[c + 1]));
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx *= a.scale_log2;
      const float m_new = fmaxf(m, mx);
      float m_use = m, corr = 1.f;
      bool rescale = false;
      if (m == -INFINITY) {
        // nothing accumulated yet (O and l are zero): start at this tile's
        // max; a row with no valid token yet keeps -inf and gets p = 0
        m_use = m_new == -INFINITY ? 0.f : m_new;
        m = m_new;
        corr = 0.f;
      } else if (m_new - m > kTcRescaleLog2) {
        m_use = m_new;
        corr = tc::ex2(m - m_new);
        rescale = true;
        m = m_new;
      }
      l *= corr;
      const float neg = -m_use;
      // p = 2^(s*scale - m) in packed pairs: 6 of every 16 columns on the
      // FMA pipe (exp2_fma2), the rest on the MUFU unit, so neither unit
      // alone limits the row; sums in two packed accumulators.
      const uint64_t scale2 = tc::pk2(a.scale_log2, a.scale_log2);
      const uint64_t neg2 = tc::pk2(neg, neg);
      uint64_t sum2[2] = {tc::pk2(0.f, 0.f), tc::pk2(0.f, 0.f)};
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const uint64_t x2 = tc::ffma2(tc::pk2(__uint_as_float(sr[64 * hf + c]),
                                                __uint_as_float(sr[64 * hf + c + 1])),
                                       scale2, neg2);
          uint64_t p2;
          if (((c >> 1) & 7) >= 5) {
            p2 = tc::exp2_fma2(x2);
          } else {
            float x0, x1;
            tc::unpk2(x2, x0, x1);
            p2 = tc::pk2(tc::ex2(x0), tc::ex2(x1));
          }
          sum2[(c >> 1) & 1] = tc::fadd2(sum2[(c >> 1) & 1], p2);
          float p0, p1;
          tc::unpk2(p2, p0, p1);
          pk[c >> 1] = tc::pack_half2(p0, p1);
        }
        // fp16 P of tokens [64hf, 64hf+64) -> columns [32hf, 32hf+32) (the
        // whole S row is already in registers)
        tc::tmem_st32(t_s + hf * 32, pk);
      }
      {
        float a0, a1, b0v, b1v;
        tc::unpk2(sum2[0], a0, a1);
        tc::unpk2(sum2[1], b0v, b1v);
        l += (a0 + a1) + (b0v + b1v);
      }
      if (__any_sync(0xffffffffu, rescale) && j > 0) {
        // O holds PV of tiles < j (PV of tile j waits for p_full below):
        // wait for the last one, then scale O in TMEM.  Done after P so the
        // S row's registers are free.
        if (!(ok = tc::mbar_wait_warp(&bars->o_full[i], (j - 1) & 1, abort_flag))) break;
        tc::fence_after_sync();
        const float f = rescale ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tc::tmem_ld32(t_o + c * 32, orr);
          tc::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) orr[q] = __float_as_uint(__uint_as_float(orr[q]) * f);
          tc::tmem_st32(t_o + c * 32, orr);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->p_full[i]);
    }
    // ---- epilogue: O / l -> bf16, LSE
    if (ok && i < nq && n_tiles > 0 &&
        tc::mbar_wait_warp(&bars->o_full[i], (n_tiles - 1) & 1, abort_flag)) {
      tc::fence_after_sync();
      const float inv_l = 1.f / l;
      bool nonfinite = false;   // inf/NaN output: V outside the fp16 range (or bad input)
      // O / l as bf16 into this Q tile's shared memory (free once its last
      // S product completed, which o_full implies), in the layout the Q load
      // used: [half][row][128 B], 128-byte swizzle; one thread then stores the
      // tile with TMA.  The store box holds at most one query block's
      // positions, and rows past the segment fall outside the tensor, so only
      // this unit's rows are written.
      char* stage = sQ + i * L::kHalves * L::kHalfBytes;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tc::tmem_ld32(t_o + c * 32, orr);
        tc::tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 pk4;
          uint32_t* pw = reinterpret_cast<uint32_t*>(&pk4);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float o0 = __uint_as_float(orr[q8 * 8 + 2 * t]) * inv_l;
            const float o1 = __uint_as_float(orr[q8 * 8 + 2 * t + 1]) * inv_l;
            nonfinite |= !(fabsf(o0) <= 3.0e38f) | !(fabsf(o1) <= 3.0e38f);
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o0, o1);
            pw[t] = *reinterpret_cast<uint32_t*>(&v2);
          }
          const int hf = (c * 32) / 64, ch = ((c * 32) % 64) / 8 + q8;   // 16-byte chunk of the row
          *reinterpret_cast<uint4*>(stage + hf * L::kHalfBytes + r * 128 + ((ch ^ (r & 7)) * 16)) = pk4;
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars->ostage[i]);
      if (quarter == 0 && lane == 0 && tc::mbar_wait(&bars->ostage[i], 0, abort_flag)) {
        const int pos_t = (int)(b0 - a.q_start) + (row0 + i * kTcRows) / a.G;
#pragma unroll
        for (int hf = 0; hf < L::kHalves; ++hf)
          tc::tma_store_3d(&tm_o, hf * 64, h * a.G, pos_t, stage + hf * L::kHalfBytes);
        tc::bulk_commit_group();
        tc::bulk_wait_group_read0();
      }
      if (row_live && a.lse)
        a.lse[(pos - a.q_start) * a.Hq + (int64_t)h * a.G + unit_row % a.G] =
            (m + log2f(l)) * 0.6931471805599453f;
      if (row_live && nonfinite) report(HGA_ERR_DEVICE_CHECK);
    }
  }

  // ---- teardown: all roles done (every wait above is bounded)
  griddep_launch();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace hga
