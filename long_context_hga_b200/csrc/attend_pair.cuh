// Step 4 on a pair of SMs: gathered exact-token attention with
// tcgen05.mma.cta_group::2 (M = 256 across the two CTAs of a cluster).
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: exact token K/V
// of the kept groups plus the sink and local windows feed softmax attention.
//
// Why a pair.  With one CTA per SM holding two 128-row Q tiles, TMEM is full
// (S0 | S1 | O0 | O1) and each tile's next S product has to wait for its P:
// the tile period is softmax + P.V + S, and the two softmax warpgroups
// alternate instead of overlapping.  Here each CTA holds ONE 128-row tile;
// the pair's MMA computes both CTAs' rows (A split by rows, B by columns), so
// every K/V byte still serves 256 rows, while each SM has TMEM for a double-
// buffered S: S(j+1) is computed during the softmax of S(j).
//
// TMEM columns (each CTA, its own 128 rows): S_a [0,128) S_b [128,256)
// O [256,384).  P (fp16) overwrites the first 64 columns of its S buffer.
//
// Each CTA loads half of every K/V tile: its 64 tokens of K (8 groups, both
// 64-dim halves) and its 64-dim half of V for all 128 tokens.  The loads
// complete on the leader CTA's barriers; the leader (rank 0) issues every
// MMA, and its commits signal both CTAs.  Padding entries of a tile are
// loaded from a group coordinate past the end of the tensor (TMA fills zeros
// and counts the bytes), so V needs no clean-up and every load moves a fixed
// 16 KB per CTA.
//
// Warp roles (384 threads per CTA):
//   warp 0      TMA producer (Q once, then K/V half tiles into a ring)
//   warp 1      TMEM allocation for the pair; in the leader, the MMA issuer
//   warp 2      waits for the last MMA before teardown
//   warps 4-7   softmax of columns 0-63 of every row (tokens 0-63 of a tile)
//   warps 8-11  softmax of columns 64-127; warps 4+q and 8+q share TMEM lane
//               quarter q and exchange their partial row maxima through
//               shared memory (one named barrier per warp pair and tile)
#pragma once
#include "attend.cuh"
#include "tc.cuh"

namespace hga {

constexpr int kPrRows = 128;               // query rows per CTA (MMA M / 2)
constexpr int kPrTok = 128;                // tokens per K/V tile (MMA N of S)
constexpr int kPrGroups = kPrTok / 8;      // 16 groups per tile
constexpr int kPrThreads = 384;
constexpr int kPrSlots = 8;                // ring of K or V half tiles
constexpr int kPrSlotBytes = 16384;        // per CTA: 8 K groups x 2 halves, or 16 V groups x 1 half
constexpr int kPrQBytes = 2 * kPrRows * 128;   // [half][128 rows][128 B]
constexpr int kPrSlotOff = kPrQBytes;
constexpr int kPrBarOff = kPrSlotOff + kPrSlots * kPrSlotBytes;
constexpr int kPrXchOff = kPrBarOff + 1024;    // floats: max [2][256], then l [256]
constexpr int kPrListOff = kPrXchOff + 3 * 256 * 4;
constexpr float kPrRescaleLog2 = 8.0f;   // rescale O only when the max grows by > 2^8

inline size_t pair_smem_bytes(int max_list) {
  return 1024 + (size_t)kPrListOff + (size_t)max_list * 4;
}

struct PrBars {
  uint64_t q_full, full[kPrSlots], empty[kPrSlots];
  uint64_t s_full[2], p_full[2], o_full, done, ostage;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PrBars) <= 1024, "barrier block");

#ifdef HGA_TIMELINE
// Debug builds only: globaltimer stamps of the first cluster's pipeline
// events, [rank][kind][tile]; kinds: 0 S issued, 1 P.V issued, 2/3 softmax
// start/end (columns 0-63), 4/5 (columns 64-127), 6 K/V load issued, 7 S
// operands ready (issue starts), 8 P and V ready (issue starts).
constexpr int kPrTlKinds = 9;
__device__ unsigned long long g_pr_ev[2 * kPrTlKinds * 128];
#define HGA_PR_TL(rank, kind, idx)                                                     \
  do {                                                                                 \
    if (blockIdx.x < 2 && blockIdx.y == 0 && blockIdx.z == 0 && (idx) < 128)           \
      g_pr_ev[((rank) * kPrTlKinds + (kind)) * 128 + (idx)] = tc::globaltimer_ns();    \
  } while (0)
// per-phase clock64 sums of the first cluster's warps 4 and 8 (lane 0),
// [rank][wg][phase]: 0 S wait, 1 TMEM load, 2 max + exchange, 3 exps + P
// store, 4 rescale + store wait, 5 arrive
__device__ unsigned long long g_pr_ph[2 * 2 * 8];
#define HGA_PR_PH(k)                                                                   \
  do {                                                                                 \
    const long long now_ = clock64();                                                  \
    ph_acc[k] += now_ - ph_t;                                                          \
    ph_t = now_;                                                                       \
  } while (0)
#else
#define HGA_PR_TL(rank, kind, idx) ((void)0)
#define HGA_PR_PH(k) ((void)0)
#endif

// The leader's MMA issuer (one thread), out of line like the single-CTA
// kernel's.  Order: S(0), S(1), then per tile j: P.V(j) once both CTAs wrote
// P(j), and S(j+2) into the buffer P(j) occupied (the tensor pipe runs them in
// order, so P.V(j) has read P before S(j+2) overwrites it).
__device__ __noinline__ void pair_mma_issuer(PrBars* bars, uint32_t tmem, uint32_t q_base,
                                             uint32_t slot_base, int n_tiles,
                                             volatile int* abort_flag) {
  constexpr uint32_t kIdS = tc::idesc_f16(256, kPrTok, 1, 0);
  constexpr uint32_t kIdPV = tc::idesc_f16(256, 128, 0, 1);
  auto both = [&](uint64_t* bar) {
    const uint32_t a = tc::smem_addr(bar);
    tc::mma2_commit(tc::map_to_rank(a, 0));
    tc::mma2_commit(tc::map_to_rank(a, 1));
  };
  // Q: [half][128 rows][128 B] (8-row groups 1 KB apart, halves 16 KB apart)
  const uint64_t q_desc = tc::sdesc_sw128(q_base, 16, 1024);
  // K half tile: [group][half][8 rows][128 B] (groups 2 KB apart, halves 1 KB)
  const uint64_t k_desc0 = tc::sdesc_sw128(slot_base, 16, 2048);
  // V half tile: [group][8 rows][128 B] (MN-major, 8-token groups 1 KB apart)
  const uint64_t v_desc0 = tc::sdesc_sw128(slot_base, 8192, 1024);
  bool ok = tc::mbar_wait(&bars->q_full, 0, abort_flag);
  tc::fence_after_sync();
  auto issue_s = [&](int j) -> bool {
    const int n = 2 * j, s = n % kPrSlots;
    if (!tc::mbar_wait(&bars->full[s], (n / kPrSlots) & 1, abort_flag)) return false;
    tc::fence_after_sync();
    HGA_PR_TL(0, 7, j);
    const uint64_t kd = k_desc0 + (uint64_t)((s * kPrSlotBytes) >> 4);
    const uint32_t d_s = tmem + (uint32_t)(j & 1) * 128;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      tc::mma2_ss(d_s, q_desc + (uint64_t)((((k >> 2) * (kPrQBytes / 2)) + (k & 3) * 32) >> 4),
                  kd + (uint64_t)((((k >> 2) * 1024) + (k & 3) * 32) >> 4), kIdS, k > 0);
    both(&bars->s_full[j & 1]);
    both(&bars->empty[s]);
    HGA_PR_TL(0, 0, j);
    return true;
  };
  auto issue_pv = [&](int j) -> bool {
    if (!tc::mbar_wait_cluster(&bars->p_full[j & 1], (j >> 1) & 1, abort_flag)) return false;
    tc::fence_after_sync();
    const int n = 2 * j + 1, s = n % kPrSlots;
    if (!tc::mbar_wait(&bars->full[s], (n / kPrSlots) & 1, abort_flag)) return false;
    tc::fence_after_sync();
    HGA_PR_TL(0, 8, j);
    const uint64_t vd = v_desc0 + (uint64_t)((s * kPrSlotBytes) >> 4);
    const uint32_t a_p = tmem + (uint32_t)(j & 1) * 128;
#pragma unroll
    for (int k = 0; k < kPrTok / 16; ++k)
      tc::mma2_ts(tmem + 256, a_p + k * 8, vd + (uint64_t)((k * 2048) >> 4), kIdPV,
                  (j > 0 || k > 0) ? 1u : 0u);
    both(&bars->o_full);
    both(&bars->empty[s]);
    HGA_PR_TL(0, 1, j);
    return true;
  };
  if (ok) ok = issue_s(0);
  if (ok && n_tiles > 1) ok = issue_s(1);
  for (int j = 0; ok && j < n_tiles; ++j) {
    ok = issue_pv(j);
    if (ok && j + 2 < n_tiles) ok = issue_s(j + 2);
  }
  both(&bars->done);   // tracks every MMA issued above
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPrThreads, 1)
    attend_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k1,
                       const __grid_constant__ CUtensorMap tm_k8,
                       const __grid_constant__ CUtensorMap tm_vh1,
                       const __grid_constant__ CUtensorMap tm_vh8,
                       const __grid_constant__ CUtensorMap tm_o, AttendArgs a) {
  static_assert(D == 128, "the pair kernel is built for d = 128");
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PrBars* bars = reinterpret_cast<PrBars*>(smem + kPrBarOff);
  float* xch = reinterpret_cast<float*>(smem + kPrXchOff);
  int* list = reinterpret_cast<int*>(smem + kPrListOff);
  volatile int* abort_flag = &bars->abort;

  griddep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_rank();
#ifdef HGA_TIMELINE
  const int cta_lin = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  if (tid == 0 && cta_lin < 4096) {
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_cta[3 * cta_lin] = tc::globaltimer_ns();
    g_cta[3 * cta_lin + 2] = smid;
  }
#endif
  const int pair = blockIdx.x >> 1;
  const int b = blockIdx.y, h = blockIdx.z;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int64_t T = a.q_start + a.n_q;
  const int npos = (int)min((int64_t)a.qblock, T - b0);
  const int nrows = npos * a.G;
  const int prow0 = pair * 2 * kPrRows;
  if (prow0 >= nrows) return;                 // the whole pair: both CTAs leave here
  const int row0 = prow0 + (int)rank * kPrRows;

  // ---- prologue: group list (each CTA its own copy), barriers, TMEM
  int n_nondiag;
  bool inv = false;
  if (tid == 0) bars->abort = 0;
  const int n_list = build_group_list(a, b, h, b0, T, list, &n_nondiag, &inv);
  if (n_list < 0) return;                     // same outcome in both CTAs
  __shared__ int s_inv;
  if (tid == 0) s_inv = 0;
  __syncthreads();
  if (inv) s_inv = 1;
  if (tid == 0) {
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kPrSlots; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&bars->s_full[x], 1);
      tc::mbar_init(&bars->p_full[x], 16);   // 8 softmax warps x 2 CTAs
    }
    tc::mbar_init(&bars->o_full, 1);
    tc::mbar_init(&bars->done, 1);
    tc::mbar_init(&bars->ostage, 256);
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(&bars->tmem_base, 512);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();                         // both CTAs' barriers exist before any remote use
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const bool any_invalid = s_inv != 0;
  const int n_tiles = (n_list + kPrGroups - 1) / kPrGroups;
  const int n_loads = 2 * n_tiles;
  char* sQ = smem;
  auto slot_ptr = [&](int s) { return smem + kPrSlotOff + s * kPrSlotBytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_q);
      tc::tma_prefetch_desc(&tm_k1);
      tc::tma_prefetch_desc(&tm_k8);
      tc::tma_prefetch_desc(&tm_vh1);
      tc::tma_prefetch_desc(&tm_vh8);
      if (rank == 0) tc::mbar_arrive_expect_tx(&bars->q_full, 2 * kPrQBytes);
    }
    __syncwarp();
    if (lane < 2) {
      const int pos0 = (int)(b0 - a.q_start) + row0 / a.G;
      tc::tma2_load_3d(sQ + lane * (kPrQBytes / 2), &tm_q, lane * 64, h * a.G, pos0,
                       tc::map_to_rank(tc::smem_addr(&bars->q_full), 0));
    }
    int last_use[kPrSlots];
#pragma unroll
    for (int s = 0; s < kPrSlots; ++s) last_use[s] = -1;
    const int64_t head_group0 = (int64_t)h * (a.t_cap / a.group);
    const int oob_group = (int)((int64_t)a.Hkv * (a.t_cap / a.group));   // zero fill
    for (int n = 0; n < n_loads; ++n) {
      const int s = n % kPrSlots, u = n / kPrSlots, j = n >> 1;
      int ok = 1;
      if (n >= kPrSlots && lane == 0) ok = tc::mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const uint32_t fbar = tc::map_to_rank(tc::smem_addr(&bars->full[s]), 0);
      if (lane == 0 && rank == 0) tc::mbar_arrive_expect_tx(&bars->full[s], 2 * kPrSlotBytes);
      __syncwarp();
      if (!(n & 1)) {
        // K: this CTA's 8 entries of tile j, [group][half][8 rows][128 B]
        const int e = lane & 7;
        const int li = j * kPrGroups + (int)rank * 8 + e;
        const int ent = li < n_list ? list[li] : -1;
        const int ent0 = __shfl_sync(0xffffffffu, ent, 0);
        const bool consec = ent >= 0 && ent0 >= 0 && ent == ent0 + e;
        const unsigned run = __ballot_sync(0xffffffffu, lane < 8 && consec) & 0xffu;
        if (run == 0xffu) {
          if (lane == 0)
            tc::tma2_load_4d(slot_ptr(s), &tm_k8, 0, 0, 0, (int)(head_group0 + ent0), fbar);
        } else if (lane < 8) {
          const int g = ent >= 0 ? (int)(head_group0 + ent) : oob_group;
          tc::tma2_load_4d(slot_ptr(s) + e * 2048, &tm_k1, 0, 0, 0, g, fbar);
        }
      } else {
        // V: all 16 entries of tile j, this CTA's 64-dim half, [group][8 rows][128 B]
        const int e = lane & 15;
        const int li = j * kPrGroups + e;
        const int ent = li < n_list ? list[li] : -1;
        const int ent0 = __shfl_sync(0xffffffffu, ent, e & ~7);
        const bool consec = ent >= 0 && ent0 >= 0 && ent == ent0 + (e & 7);
        const unsigned cm = __ballot_sync(0xffffffffu, lane < 16 && consec);
        const bool run = ((cm >> (e & ~7)) & 0xffu) == 0xffu;
        if (lane < 16) {
          if (run) {
            if ((e & 7) == 0)
              tc::tma2_load_4d(slot_ptr(s) + e * 1024, &tm_vh8, 0, 0, (int)rank,
                               (int)(head_group0 + ent), fbar);
          } else {
            const int g = ent >= 0 ? (int)(head_group0 + ent) : oob_group;
            tc::tma2_load_4d(slot_ptr(s) + e * 1024, &tm_vh1, 0, 0, (int)rank, g, fbar);
          }
        }
      }
      last_use[s] = u;
      if (lane == 0) HGA_PR_TL(rank, 6, n);
    }
    // the leader's full barriers count both CTAs' bytes: once they have all
    // landed, no copy is still writing into either CTA's shared memory
    if (lane == 0 && rank == 0) {
      for (int s = 0; s < kPrSlots; ++s) {
        if (last_use[s] < 0) continue;
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&bars->full[s], last_use[s] & 1) &&
               tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0)
      pair_mma_issuer(bars, tmem, tc::smem_addr(sQ), tc::smem_addr(slot_ptr(0)), n_tiles,
                      abort_flag);
  } else if (warp == 2) {
    // ------------------------------------------------------------ drain
    // every MMA of the pair (they read this CTA's shared memory and write its
    // TMEM) has completed before teardown
    if (lane == 0) tc::mbar_wait(&bars->done, 0, abort_flag);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;           // 0: columns 0-63, 1: columns 64-127
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;        // TMEM lane = row of this CTA's tile
    const int unit_row = row0 + r;
    const bool row_live = unit_row < nrows;
    const int64_t pos = b0 + (row_live ? unit_row / a.G : 0);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_o = tmem + lane_off + 256 + wg * 64;
    const uint32_t pfull[2] = {tc::map_to_rank(tc::smem_addr(&bars->p_full[0]), 0),
                               tc::map_to_rank(tc::smem_addr(&bars->p_full[1]), 0)};
    const int bar_id = 1 + quarter;           // warps 4+q and 8+q
    float m = -INFINITY, l = 0.f;
    bool ok = true;
#ifdef HGA_TIMELINE
    long long ph_acc[6] = {0, 0, 0, 0, 0, 0};
    long long ph_t = clock64();
#endif
    for (int j = 0; j < n_tiles; ++j) {
      const int x = j & 1;
      if (ok) ok = tc::mbar_wait(&bars->s_full[x], (j >> 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);       // warp-uniform from here on
      HGA_PR_PH(0);
      if (lane == 0 && quarter == 0) HGA_PR_TL(rank, 2 + 2 * wg, j);
      tc::fence_after_sync();
      const uint32_t t_s = tmem + lane_off + (uint32_t)x * 128;
      uint32_t sr[64];
      if (ok) {
        tc::tmem_ld32(t_s + wg * 64, sr);
        tc::tmem_ld32(t_s + wg * 64 + 32, sr + 32);
        tc::tmem_wait_ld();
        HGA_PR_PH(1);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) sr[c] = __float_as_uint(-INFINITY);
      }
      const bool need_mask =
          any_invalid || (j * kPrGroups + (wg + 1) * 8 > n_nondiag);
      if (need_mask) {
        const int pos32 = (int)pos;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int li = j * kPrGroups + wg * 8 + e;
          const int ent = li < n_list ? list[li] : -1;
          const int lim = ent < 0 ? -1 : pos32 - ent * 8;   // valid columns c <= lim
#pragma unroll
          for (int c = 0; c < 8; ++c)
            if (c > lim) sr[e * 8 + c] = __float_as_uint(-INFINITY);
        }
      }
      float mx4[4];
#pragma unroll
      for (int x4 = 0; x4 < 4; ++x4) mx4[x4] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 2)
        mx4[(c >> 1) & 3] = tc::fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]),
                                      __uint_as_float(sr[c + 1]));
      float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      // partner half of the row (same TMEM lane, other warpgroup)
      xch[x * 256 + wg * 128 + r] = mx;
      asm volatile("bar.sync %0, 64;\n" ::"r"(bar_id) : "memory");
      mx = fmaxf(mx, xch[x * 256 + (1 - wg) * 128 + r]) * a.scale_log2;
      HGA_PR_PH(2);
      if (!ok) continue;
      const float m_new = fmaxf(m, mx);
      float m_use = m, corr = 1.f;
      bool rescale = false;
      if (m == -INFINITY) {
        m_use = m_new == -INFINITY ? 0.f : m_new;
        m = m_new;
        corr = 0.f;
      } else if (m_new - m > kPrRescaleLog2) {
        m_use = m_new;
        corr = tc::ex2(m - m_new);
        rescale = true;
        m = m_new;
      }
      l *= corr;
      const float neg = -m_use;
      const uint64_t scale2 = tc::pk2(a.scale_log2, a.scale_log2);
      const uint64_t neg2 = tc::pk2(neg, neg);
      uint64_t sum2[2] = {tc::pk2(0.f, 0.f), tc::pk2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const uint64_t x2 = tc::ffma2(
            tc::pk2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), scale2, neg2);
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
      // fp16 P of this half's 64 tokens -> columns [32 wg, 32 wg + 32) of the
      // S buffer (the partner has read its S columns before the barrier)
      tc::tmem_st32(t_s + wg * 32, pk);
      HGA_PR_PH(3);
      {
        float a0, a1, b0v, b1v;
        tc::unpk2(sum2[0], a0, a1);
        tc::unpk2(sum2[1], b0v, b1v);
        l += (a0 + a1) + (b0v + b1v);
      }
      if (__any_sync(0xffffffffu, rescale) && j > 0) {
        // O holds P.V of tiles < j; P.V(j) waits for this warp's arrival below
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->o_full, (j - 1) & 1, abort_flag));
        if (!ok) continue;
        tc::fence_after_sync();
        const float f = rescale ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
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
      __syncwarp();
      HGA_PR_PH(4);
      if (lane == 0) tc::mbar_arrive_cluster(pfull[x]);
      HGA_PR_PH(5);
      if (lane == 0 && quarter == 0) HGA_PR_TL(rank, 3 + 2 * wg, j);
    }
#ifdef HGA_TIMELINE
    if (blockIdx.x < 2 && blockIdx.y == 0 && blockIdx.z == 0 && lane == 0 && quarter == 0)
      for (int k = 0; k < 6; ++k) g_pr_ph[(rank * 2 + wg) * 8 + k] = ph_acc[k] / max(1, n_tiles);
#endif
    // ---- epilogue: O / l -> bf16 through shared memory, TMA stores, LSE
    if (ok) ok = tc::mbar_wait(&bars->o_full, (n_tiles - 1) & 1, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    tc::fence_after_sync();
    xch[512 + wg * 128 + r] = l;
    asm volatile("bar.sync %0, 64;\n" ::"r"(bar_id) : "memory");
    const float l_row = l + xch[512 + (1 - wg) * 128 + r];
    if (ok) {
      const float inv_l = 1.f / l_row;
      bool nonfinite = false;
      // this half's 64 output dims -> half wg of the (now free) Q tile, in the
      // layout the Q load used: [half][row][128 B], 128-byte swizzle
      char* stage = sQ + wg * (kPrQBytes / 2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
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
          const int ch = c * 4 + q8;   // 16-byte chunk of the 128-byte row
          *reinterpret_cast<uint4*>(stage + r * 128 + ((ch ^ (r & 7)) * 16)) = pk4;
        }
      }
      if (row_live && nonfinite) report(HGA_ERR_DEVICE_CHECK);
      if (wg == 0 && row_live && a.lse)
        a.lse[(pos - a.q_start) * a.Hq + (int64_t)h * a.G + unit_row % a.G] =
            (m + log2f(l_row)) * 0.6931471805599453f;
    }
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars->ostage);
    if (warp == 4 && lane == 0 && ok && tc::mbar_wait(&bars->ostage, 0, abort_flag)) {
      const int pos_t = (int)(b0 - a.q_start) + row0 / a.G;
      tc::tma_store_3d(&tm_o, 0, h * a.G, pos_t, sQ);
      tc::tma_store_3d(&tm_o, 64, h * a.G, pos_t, sQ + kPrQBytes / 2);
      tc::bulk_commit_group();
      tc::bulk_wait_group_read0();
    }
  }

  // ---- teardown: all roles done (every wait above is bounded); neither CTA
  // leaves while the pair's MMAs or copies may still touch its memory
  griddep_launch();
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, 512);
  }
#ifdef HGA_TIMELINE
  if (tid == 0 && cta_lin < 4096) g_cta[3 * cta_lin + 1] = tc::globaltimer_ns();
#endif
}

}  // namespace hga
