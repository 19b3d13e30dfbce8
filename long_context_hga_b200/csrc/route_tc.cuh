// Steps 2 and 3 on the sm_100a tensor cores: chunk / group routing with
// tcgen05.mma and TMEM accumulators.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: the query block
// scores the summaries and keeps the best chunks, then the best groups inside
// them; one decision per (query block, KV head) (section 6.1).
//
// One CTA per (query block, KV head).  The score of a candidate is a max over
// the block's rows, so the product is computed transposed,
//   D[candidate][row] = summary[candidate] . q[row]   (M = 128 candidates,
//                                                       N = up to 256 rows),
// which puts one candidate in each TMEM lane: an epilogue thread reduces its
// own lane's columns in registers, no cross-thread reduction.  Rows are staged
// once (TMA, 128-byte swizzle); candidate summaries stream through a 2-stage
// TMA ring of 8-row boxes (8 consecutive chunks, or the 8 groups of one kept
// chunk).  The TMEM accumulator is double buffered (2 x up to 256 columns) so
// the epilogue of one (tile, row slice) overlaps the product of the next.
//
// Warps (256 threads): 0 TMA producer, 1 TMEM owner + MMA issuer, 4-7
// epilogue (TMEM lane quarters 0-3); afterwards all 256 threads run the exact
// radix selection of route.cuh (score desc, index asc).
#pragma once
#include "route.cuh"
#include "tc.cuh"

namespace hga {

constexpr int kRtThreads = 256;
constexpr int kRtTile = 128;                // candidates per tile (MMA M)
constexpr int kRtMaxCands = 4096;           // shared-memory score slots
constexpr int kRtMaxRows = 512;             // query rows per unit (G <= 8)

template <int D>
struct RtLayout {
  static constexpr int kHalves = D / 64;
  static constexpr int kQHalf = 256 * 128;                       // rows x 128 B
  static constexpr int kQBytes = 2 * kHalves * kQHalf;           // up to 2 slices of 256
  static constexpr int kTileHalf = kRtTile * 128;                // 16 KB
  static constexpr int kStageBytes = kHalves * kTileHalf;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kScoreOff = kStageOff + 2 * kStageBytes;
  static constexpr int kBarOff = kScoreOff + kRtMaxCands * 4;
  static constexpr size_t kSmem = 1024 + (size_t)kBarOff + 256;   // 2 barrier sets
};

struct RtBars {
  uint64_t q_full, full[2], empty[2], acc_full[2], acc_empty[2], done;
  uint32_t tmem_base;
  int abort;
};


struct RtArgs {
  RouteArgs r;
  int rs;            // query rows per slice (MMA N): min(256, 64 * G)
};

// Scores every candidate of `cd` for the unit (block at b0, KV head h):
// sc[i] = max over the unit's rows of q_row . summary(cd.id(i)).  Warp 0
// streams the summaries (and Q first when load_q, unless q_issued: the caller
// then initialised q_full and requested Q itself; without load_q Q is already
// in shared memory), warp 1 issues the MMAs into the double-buffered TMEM
// accumulator at `tmem`, warps 4-7 reduce each candidate's row maxima.  Uses
// the barrier set `bars` (initialised here) and ends with a CTA barrier.
template <int D>
__device__ void rt_score(const CUtensorMap* tm_q, const CUtensorMap* tm_s, bool load_q, bool q_issued,
                         const RouteArgs& a, const Cands& cd, int RS, int nrows, int64_t b0,
                         int h, char* smem, RtBars* bars, uint32_t tmem, float* sc,
                         volatile int* abort_flag) {
  using L = RtLayout<D>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_slices = (nrows + RS - 1) / RS;
  const int n_tiles = (cd.n + kRtTile - 1) / kRtTile;
  const int n_jobs = n_tiles * n_slices;
  if (tid == 0) {
    if (!q_issued) tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
      tc::mbar_init(&bars->acc_full[s], 1);
      tc::mbar_init(&bars->acc_empty[s], 128);
    }
    tc::mbar_init(&bars->done, 1);
    tc::fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  char* sQ = smem;
  auto stage = [&](int s, int hf) { return smem + L::kStageOff + s * L::kStageBytes + hf * L::kTileHalf; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Q once; then candidate summaries per 128-candidate tile: in chunk mode
    // the tile's rows are contiguous and come as one 128-row box per 64-dim
    // half; in group mode each kept chunk's 8 groups are one 8-row box per
    // half (lane e < 16 issues kept chunk e of the tile).
    if (lane == 0) {
      tc::tma_prefetch_desc(tm_s);
      if (load_q && !q_issued) {
        tc::tma_prefetch_desc(tm_q);
        const int pos0 = (int)(b0 - a.q_start);
        tc::mbar_arrive_expect_tx(&bars->q_full, n_slices * L::kHalves * RS * 128);
        for (int r = 0; r < n_slices; ++r)
          for (int hf = 0; hf < L::kHalves; ++hf)
            tc::tma_load_3d(sQ + (r * L::kHalves + hf) * L::kQHalf, tm_q, hf * 64, h * a.G,
                            pos0 + r * (RS / a.G), &bars->q_full);
      }
    }
    int pending[2] = {-1, -1};
    const int row_head = (int)((int64_t)h * a.n_summ_cap);
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1, u = t >> 1;
      int ok = 1;
      if (t >= 2 && lane == 0) ok = tc::mbar_wait(&bars->empty[s], (u - 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (!a.group_mode) {
        if (lane == 0) {
          tc::mbar_arrive_expect_tx(&bars->full[s], L::kHalves * L::kTileHalf);
          for (int hf = 0; hf < L::kHalves; ++hf)
            tc::tma_load_2d(stage(s, hf), tm_s, hf * 64, row_head + cd.lo + t * kRtTile,
                            &bars->full[s]);
        }
      } else {
        const int n_box = min(kRtTile / 8, (cd.n - t * kRtTile + 7) / 8);
        if (lane == 0) tc::mbar_arrive_expect_tx(&bars->full[s], n_box * L::kHalves * 1024);
        __syncwarp();
        if (lane < n_box) {
          const int row = row_head + cd.kept[t * (kRtTile / 8) + lane] * cd.per;
          for (int hf = 0; hf < L::kHalves; ++hf)
            tc::tma_load_2d(stage(s, hf) + lane * 1024, tm_s, hf * 64, row, &bars->full[s]);
        }
      }
      pending[s] = u;
    }
    if (lane == 0) {
      for (int s = 0; s < 2; ++s) {
        if (pending[s] < 0) continue;
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&bars->full[s], pending[s] & 1) &&
               tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA
      // the whole warp runs the loop; elect.sync picks the issuing lane
      const uint32_t idesc = tc::idesc_f16(kRtTile, RS, 1, 0);
      const uint32_t q_base = tc::smem_addr(sQ);
      bool ok = !load_q || tc::mbar_wait_warp(&bars->q_full, 0, abort_flag);
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t & 1;
        if (!(ok = tc::mbar_wait_warp(&bars->full[s], (t >> 1) & 1, abort_flag))) break;
        tc::fence_after_sync();
        for (int r = 0; r < n_slices; ++r) {
          const int q = t * n_slices + r, buf = q & 1;
          if (q >= 2 &&
              !(ok = tc::mbar_wait_warp(&bars->acc_empty[buf], ((q >> 1) - 1) & 1, abort_flag)))
            break;
          tc::fence_after_sync();
          // base descriptors once; k-steps move only the start address
          const uint64_t ad0 = tc::sdesc_sw128(tc::smem_addr(stage(s, 0)), 16, 1024);
          const uint64_t bd0 = tc::sdesc_sw128(q_base + r * L::kHalves * L::kQHalf, 16, 1024);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            tc::mma_ss_warp(tmem + buf * 256,
                            ad0 + (uint64_t)((((k >> 2) * L::kTileHalf) + (k & 3) * 32) >> 4),
                            bd0 + (uint64_t)((((k >> 2) * L::kQHalf) + (k & 3) * 32) >> 4), idesc,
                            k > 0);
          tc::mma_commit_warp(&bars->acc_full[buf]);
        }
        if (ok) tc::mma_commit_warp(&bars->empty[s]);
      }
      tc::mma_commit_warp(&bars->done);
      const uint64_t t0 = tc::globaltimer_ns();
      while (!tc::mbar_try_wait(&bars->done, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int cl = quarter * 32 + lane;                 // candidate lane in the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float best = -INFINITY;
    for (int q = 0; q < n_jobs; ++q) {
      const int t = q / n_slices, r = q % n_slices, buf = q & 1;
      if (!tc::mbar_wait(&bars->acc_full[buf], (q >> 1) & 1, abort_flag)) break;
      tc::fence_after_sync();
      const int valid_cols = min(RS, nrows - r * RS);    // rows past the block: masked
      // up to 128 columns in flight per TMEM round trip (RS is 64, 128 or 256)
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      for (int c0 = 0; c0 < RS; c0 += 128) {
        uint32_t v[128];
        const int nld = min(128, RS - c0) / 32;
#pragma unroll
        for (int x = 0; x < 4; ++x)
          if (x < nld) tc::tmem_ld32(tmem + lane_off + buf * 256 + c0 + 32 * x, v + 32 * x);
        tc::tmem_wait_ld();
        if (c0 + 128 <= valid_cols && nld == 4) {
#pragma unroll
          for (int x = 0; x < 128; x += 2)
            m4[(x >> 1) & 3] = tc::fmax3(m4[(x >> 1) & 3], __uint_as_float(v[x]), __uint_as_float(v[x + 1]));
        } else {
#pragma unroll
          for (int x = 0; x < 128; ++x)
            if (x < 32 * nld && c0 + x < valid_cols) m4[x & 3] = fmaxf(m4[x & 3], __uint_as_float(v[x]));
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->acc_empty[buf]);
      best = fmaxf(best, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
      if (r == n_slices - 1) {
        const int i = t * kRtTile + cl;
        if (i < cd.n) sc[i] = best;
        best = -INFINITY;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
}

// Chunk routing or group routing of one (query block, KV head) unit.  QE:
// the call's q_early (a compile-time choice, so that the default form is
// built without the early-copy code).
template <int D, bool QE>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_s,
                    const __grid_constant__ CUtensorMap tm_s8, RtArgs args) {
  using L = RtLayout<D>;
  const RouteArgs& a = args.r;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RtBars* bars = reinterpret_cast<RtBars*>(smem + L::kBarOff);
  float* sc = reinterpret_cast<float*>(smem + L::kScoreOff);
  volatile int* abort_flag = &bars->abort;
  __shared__ int s_kept[2048];
  __shared__ int s_nkept;
  __shared__ int hist[256];
  __shared__ int tmp[32 + 256];          // scan slots + second histogram buffer

  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.x, h = blockIdx.y;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int npos = (int)min((int64_t)a.qblock, a.q_start + a.n_q - b0);
  const int nrows = npos * a.G;
  // With q_early, Q (an input of the call, complete before the previous
  // kernel can let this one start) is requested before waiting for that
  // kernel, so its load overlaps the previous kernel's tail; exits that score
  // nothing then wait for that copy first.
  constexpr bool q_issued = QE;
  if (QE && tid == 0) {
    const int RS = args.rs, n_slices = (nrows + RS - 1) / RS;
    tc::mbar_init(&bars->q_full, 1);
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&tm_q);
    tc::mbar_arrive_expect_tx(&bars->q_full, n_slices * L::kHalves * RS * 128);
    for (int r = 0; r < n_slices; ++r)
      for (int hf = 0; hf < L::kHalves; ++hf)
        tc::tma_load_3d(smem + (r * L::kHalves + hf) * L::kQHalf, &tm_q, hf * 64, h * a.G,
                        (int)(b0 - a.q_start) + r * (RS / a.G), &bars->q_full);
  }
  auto drain_q = [&]() {
    if (QE && tid == 0) {
      const uint64_t t0 = tc::globaltimer_ns();
      while (!tc::mbar_try_wait(&bars->q_full, 0) &&
             tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
      }
    }
  };
  griddep_wait();

  // ---- candidates (same rules as route_kernel)
  Cands cd;
  cd.kept = nullptr;
  cd.per = a.chunk / a.group;
  cd.lo = a.sink / a.chunk;
  const int64_t hi = b0 - a.local > 0 ? (b0 - a.local) / a.chunk : 0;
  if (!a.group_mode) {
    cd.n = hi > cd.lo ? (int)(hi - cd.lo) : 0;
  } else {
    cd.n = compact_kept_chunks(a, b, h, cd.lo, hi, s_kept, &s_nkept, tmp) * cd.per;
    cd.kept = s_kept;
  }
  const int k_eff = a.top_k <= 0 ? cd.n : min(a.top_k, cd.n);
  int32_t* out = a.out_idx + ((int64_t)h * a.n_blocks + b) * a.out_cap;
  if (k_eff > a.out_cap || cd.n > kRtMaxCands) {
    if (tid == 0) report(HGA_ERR_DEVICE_CHECK);
    drain_q();
    return;
  }
  for (int i = k_eff + tid; i < a.out_cap; i += kRtThreads) out[i] = -1;
  if (tid == 0) a.out_cnt[(int64_t)h * a.n_blocks + b] = k_eff;
  if (k_eff == 0) {
    drain_q();
    return;
  }
  if (k_eff >= cd.n) {          // every candidate kept: no scores needed
    select_emit(sc, cd, k_eff, out, hist, tmp);
    drain_q();
    return;
  }

  // ---- scoring on the tensor cores
  if (tid == 0) bars->abort = 0;
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  rt_score<D>(&tm_q, a.group_mode ? &tm_s8 : &tm_s, true, q_issued, a, cd, args.rs, nrows, b0, h, smem, bars,
              tmem, sc, abort_flag);
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
  if (*abort_flag) return;
  griddep_launch();
  select_emit(sc, cd, k_eff, out, hist, tmp);
}

struct RtFusedArgs {
  RouteArgs c;       // chunk routing (chunk summaries)
  RouteArgs g;       // group routing (group summaries); in_idx/in_cnt unused
  int rs;
};

// Chunk routing then group routing of one unit in one CTA: the block's rows
// are staged once, the kept chunks go from the first selection straight into
// the second scoring pass, and one TMEM allocation serves both.  Writes the
// same chunk_idx/chunk_cnt and group_idx/group_cnt as the two-kernel path.
template <int D>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_c,
                          const __grid_constant__ CUtensorMap tm_g8, RtFusedArgs args) {
  using L = RtLayout<D>;
  const RouteArgs& ac = args.c;
  const RouteArgs& ag = args.g;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RtBars* bars = reinterpret_cast<RtBars*>(smem + L::kBarOff);      // 2 sets: chunks, groups
  float* sc = reinterpret_cast<float*>(smem + L::kScoreOff);
  volatile int* abort_flag = &bars[0].abort;
  __shared__ int s_kept[2048];
  __shared__ int hist[256];
  __shared__ int tmp[32 + 256];          // scan slots + second histogram buffer

  const int tid = threadIdx.x, warp = tid >> 5;
  griddep_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int64_t b0 = ac.q_start + (int64_t)b * ac.qblock;
  const int npos = (int)min((int64_t)ac.qblock, ac.q_start + ac.n_q - b0);
  const int nrows = npos * ac.G;
  const int per = ac.chunk / ac.group;

  // ---- chunk candidates
  Cands cc;
  cc.kept = nullptr;
  cc.per = per;
  cc.lo = ac.sink / ac.chunk;
  const int64_t hi = b0 - ac.local > 0 ? (b0 - ac.local) / ac.chunk : 0;
  cc.n = hi > cc.lo ? (int)(hi - cc.lo) : 0;
  const int k_c = ac.top_k <= 0 ? cc.n : min(ac.top_k, cc.n);
  int32_t* out_c = ac.out_idx + ((int64_t)h * ac.n_blocks + b) * ac.out_cap;
  int32_t* out_g = ag.out_idx + ((int64_t)h * ag.n_blocks + b) * ag.out_cap;
  const int n_g = k_c * per;
  const int k_g = ag.top_k <= 0 ? n_g : min(ag.top_k, n_g);
  if (k_c > ac.out_cap || cc.n > kRtMaxCands || k_c > 2048 || n_g > kRtMaxCands ||
      k_g > ag.out_cap) {
    if (tid == 0) report(HGA_ERR_DEVICE_CHECK);
    return;
  }
  for (int i = k_c + tid; i < ac.out_cap; i += kRtThreads) out_c[i] = -1;
  for (int i = k_g + tid; i < ag.out_cap; i += kRtThreads) out_g[i] = -1;
  if (tid == 0) {
    ac.out_cnt[(int64_t)h * ac.n_blocks + b] = k_c;
    ag.out_cnt[(int64_t)h * ag.n_blocks + b] = k_g;
  }
  if (k_c == 0) return;
  const bool score_c = k_c < cc.n, score_g = k_g < n_g;

  if (tid == 0) bars[0].abort = 0;
  if (score_c || score_g) {
    if (warp == 1) {
      tc::tmem_alloc(&bars[0].tmem_base, 512);
      tc::tmem_relinquish();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars[0].tmem_base;
  // ---- chunk scores and selection
  if (score_c)
    rt_score<D>(&tm_q, &tm_c, true, false, ac, cc, args.rs, nrows, b0, h, smem, &bars[0], tmem, sc,
                abort_flag);
  if (*abort_flag) {
    if ((score_c || score_g) && warp == 1) tc::tmem_dealloc(tmem, 512);
    return;
  }
  select_emit(sc, cc, k_c, out_c, hist, tmp);
  __syncthreads();                       // this CTA's chunk_idx writes are visible to it
  // ---- the kept chunks' groups: scores and selection
  for (int i = tid; i < k_c; i += kRtThreads) s_kept[i] = out_c[i];
  __syncthreads();
  Cands cg;
  cg.kept = s_kept;
  cg.per = per;
  cg.lo = cc.lo;
  cg.n = n_g;
  if (score_g)
    rt_score<D>(&tm_q, &tm_g8, !score_c, false, ag, cg, args.rs, nrows, b0, h, smem, &bars[1], tmem, sc,
                abort_flag);
  if ((score_c || score_g) && warp == 1) tc::tmem_dealloc(tmem, 512);
  if (*abort_flag) return;
  griddep_launch();
  select_emit(sc, cg, k_g, out_g, hist, tmp);
}

}  // namespace hga
