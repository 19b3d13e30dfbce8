// Steps 2 and 3: chunk routing and group routing.
//
// "Long-Context Fine-Tuning with Limited VRAM", section 2.1: the current query
// block scores the chunk summaries and keeps the most relevant chunks (besides
// the sink and local windows); the kept chunks are then opened and the best
// groups inside them are kept.  Section 6.1: one decision per block.
//
// One CTA per (query block, KV head).  The block's rows (64 positions x the G
// query heads of the KV head) are staged in shared memory; candidate
// summaries stream through a double-buffered cp.async ring, 64 at a time.
// The score tile rows x 64 is a dense contraction over d and runs on the
// tensor cores (bf16 x bf16 -> fp32, mma.sync m16n8k16); its epilogue reduces
// each column to its max over the rows (warp shuffles, then across warps in
// shared memory).  The fp32 configuration uses exact FFMA dot products.
// Selection is an exact radix select over 64-bit keys (score, ~index), so
// equal scores go to the lower index; the kept candidates are emitted in
// ascending index order with a block-wide scan.
#pragma once
#include "common.cuh"

namespace hga {

constexpr int kRouteThreads = 256;
constexpr int kRouteTile = 64;          // candidates per smem tile
constexpr int kRouteMaxRowsBf16 = 256;  // query rows staged per slice (bf16)
constexpr int kRouteMaxRowsF32 = 128;   // query rows staged per slice (fp32)

struct RouteArgs {
  const void* q;          // [n_q][Hq][D]
  int64_t q_start, n_q;
  const void* summ;       // chunk_sum or group_sum, [Hkv][n_summ_cap][D]
  int64_t n_summ_cap;     // t_cap/chunk or t_cap/group
  const int32_t* in_idx;  // group mode: chunk_idx; chunk mode: unused
  const int32_t* in_cnt;
  int64_t in_cap;         // slots per (h, b) of in_idx
  int32_t* out_idx;
  int32_t* out_cnt;
  int64_t out_cap;
  int n_blocks, Hq, Hkv, G;
  int chunk, group, qblock, sink, local;
  int top_k;              // <= 0: all
  int group_mode;         // 0: chunk candidates, 1: groups of kept chunks
  int max_cands;          // shared-memory score slots
  int q_early;            // q may be requested before waiting for the previous kernel
};

// ---------------------------------------------------------------- block scan

// Exclusive prefix sum over the CTA (256 threads); returns the total in *total.
__device__ __forceinline__ int block_excl_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < kRouteThreads / 32 ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kRouteThreads / 32) tmp[lane] = t;   // inclusive warp totals
  }
  __syncthreads();
  int base = w > 0 ? tmp[w - 1] : 0;
  *total = tmp[kRouteThreads / 32 - 1];
  __syncthreads();
  return base + x - v;
}

// ---------------------------------------------------------------- mma.sync

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                        uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float* c, const uint32_t* a, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// Byte offset of the 16-byte chunk `ch` of row `r` in a [rows][D] bf16 tile
// whose chunks are XOR-swizzled by the row's low 3 bits (conflict-free
// ldmatrix on rows 2*D bytes apart).
template <int D>
__device__ __forceinline__ int swz(int r, int ch) {
  return r * (D * 2) + ((ch ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------- candidates

// Candidate ids of (b, h) are produced on the fly: chunk mode -> lo + i;
// group mode -> kept_chunk[i / per] * per + i % per, from a compacted smem list.
struct Cands {
  int n;
  int lo;           // chunk mode
  const int* kept;  // group mode (smem)
  int per;
  __device__ __forceinline__ int id(int i) const {
    return kept ? kept[i / per] * per + (i % per) : lo + i;
  }
};

// ---------------------------------------------------------------- scoring

// bf16 scores via mma.sync: sc[i] = max over rows of q_row . summ[id(i)].
template <int D>
__device__ void score_bf16(const RouteArgs& a, int b, int h, int b0, int nrows,
                           const Cands& cd, float* sc, char* smem_q,
                           char* smem_tiles, float* red) {
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* summ = reinterpret_cast<const __nv_bfloat16*>(a.summ) +
                              (int64_t)h * a.n_summ_cap * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  const int n_tiles = (cd.n + kRouteTile - 1) / kRouteTile;
  const int64_t row_stride = (int64_t)a.Hq * D;
  const __nv_bfloat16* qblk = q + (int64_t)(b0 - a.q_start) * row_stride + (int64_t)h * a.G * D;

  for (int i = tid; i < cd.n; i += kRouteThreads) sc[i] = -INFINITY;

  for (int r_lo = 0; r_lo < nrows; r_lo += kRouteMaxRowsBf16) {
    const int r_n = min(kRouteMaxRowsBf16, nrows - r_lo);
    const int r_pad = (r_n + 31) & ~31;
    __syncthreads();
    // stage the row slice (zero-filled up to a multiple of 32 rows)
    for (int e = tid; e < r_pad * kChunks; e += kRouteThreads) {
      const int r = e / kChunks, ch = e % kChunks;
      const int rr = r_lo + r;
      const __nv_bfloat16* src = qblk + (int64_t)(rr / a.G) * row_stride + (rr % a.G) * D + ch * 8;
      cp_async16(smem_u32(smem_q + swz<D>(r, ch)), r < r_n ? src : qblk, r < r_n ? 16 : 0);
    }
    auto load_tile = [&](int t, int buf) {
      char* dst = smem_tiles + buf * (kRouteTile * D * 2);
      for (int e = tid; e < kRouteTile * kChunks; e += kRouteThreads) {
        const int r = e / kChunks, ch = e % kChunks;
        const int i = t * kRouteTile + r;
        const bool ok = i < cd.n;
        const __nv_bfloat16* src = summ + (int64_t)(ok ? cd.id(i) : 0) * D + ch * 8;
        cp_async16(smem_u32(dst + swz<D>(r, ch)), src, ok ? 16 : 0);
      }
    };
    load_tile(0, 0);
    cp_async_commit();
    for (int t = 0; t < n_tiles; ++t) {
      if (t + 1 < n_tiles) load_tile(t + 1, (t + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const char* tile = smem_tiles + (t & 1) * (kRouteTile * D * 2);
      // per-lane running column max for cols nt*8 + 2*(lane%4) + {0,1}
      float cmax[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) cmax[i] = -INFINITY;
      for (int rc = warp; rc * 32 < r_pad; rc += kRouteThreads / 32) {
        float acc[2][8][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t af[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int r = rc * 32 + mt * 16 + (lane & 15);
            const int ch = kk * 2 + (lane >> 4);
            ldsm_x4(smem_u32(smem_q + swz<D>(r, ch)), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
          }
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
            const int ch = kk * 2 + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(smem_u32(tile + swz<D>(r, ch)), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              mma_bf16(acc[mt][2 * np], af[mt], b0, b1);
              mma_bf16(acc[mt][2 * np + 1], af[mt], b2, b3);
            }
          }
        }
        const int g = lane >> 2;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const bool v0 = rc * 32 + mt * 16 + g < r_n;
          const bool v1 = rc * 32 + mt * 16 + g + 8 < r_n;
#pragma unroll
          for (int nt = 0; nt < 8; ++nt) {
            float x0 = fmaxf(v0 ? acc[mt][nt][0] : -INFINITY, v1 ? acc[mt][nt][2] : -INFINITY);
            float x1 = fmaxf(v0 ? acc[mt][nt][1] : -INFINITY, v1 ? acc[mt][nt][3] : -INFINITY);
            cmax[2 * nt] = fmaxf(cmax[2 * nt], x0);
            cmax[2 * nt + 1] = fmaxf(cmax[2 * nt + 1], x1);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float x = cmax[i];
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
        cmax[i] = x;
      }
      if (lane < 4) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          red[warp * kRouteTile + nt * 8 + 2 * lane] = cmax[2 * nt];
          red[warp * kRouteTile + nt * 8 + 2 * lane + 1] = cmax[2 * nt + 1];
        }
      }
      __syncthreads();
      if (tid < kRouteTile) {
        const int i = t * kRouteTile + tid;
        if (i < cd.n) {
          float m = sc[i];
#pragma unroll
          for (int w = 0; w < kRouteThreads / 32; ++w) m = fmaxf(m, red[w * kRouteTile + tid]);
          sc[i] = m;
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
  }
  __syncthreads();
}

// fp32 scores with exact FFMA dot products (the fp32 configuration).
template <int D>
__device__ void score_f32(const RouteArgs& a, int b, int h, int b0, int nrows,
                          const Cands& cd, float* sc, float* sq, float* stile,
                          float* red) {
  const float* q = reinterpret_cast<const float*>(a.q);
  const float* summ = reinterpret_cast<const float*>(a.summ) + (int64_t)h * a.n_summ_cap * D;
  const int tid = threadIdx.x;
  const int64_t row_stride = (int64_t)a.Hq * D;
  const float* qblk = q + (int64_t)(b0 - a.q_start) * row_stride + (int64_t)h * a.G * D;
  for (int i = tid; i < cd.n; i += kRouteThreads) sc[i] = -INFINITY;
  for (int r_lo = 0; r_lo < nrows; r_lo += kRouteMaxRowsF32) {
    const int r_n = min(kRouteMaxRowsF32, nrows - r_lo);
    __syncthreads();
    for (int e = tid; e < r_n * D; e += kRouteThreads) {
      const int r = e / D, c = e % D, rr = r_lo + r;
      sq[r * (D + 1) + c] = qblk[(int64_t)(rr / a.G) * row_stride + (rr % a.G) * D + c];
    }
    for (int t0 = 0; t0 < cd.n; t0 += kRouteTile) {
      __syncthreads();
      for (int e = tid; e < kRouteTile * D; e += kRouteThreads) {
        const int r = e / D, c = e % D, i = t0 + r;
        stile[r * (D + 1) + c] = i < cd.n ? summ[(int64_t)cd.id(i) * D + c] : 0.f;
      }
      __syncthreads();
      const int col = tid % kRouteTile, rg = tid / kRouteTile;  // 4 row groups
      float m = -INFINITY;
      for (int r = rg; r < r_n; r += kRouteThreads / kRouteTile) {
        float acc = 0.f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) acc = fmaf(sq[r * (D + 1) + c], stile[col * (D + 1) + c], acc);
        m = fmaxf(m, acc);
      }
      red[rg * kRouteTile + col] = m;
      __syncthreads();
      if (tid < kRouteTile && t0 + tid < cd.n) {
        float x = sc[t0 + tid];
        for (int w = 0; w < kRouteThreads / kRouteTile; ++w) x = fmaxf(x, red[w * kRouteTile + tid]);
        sc[t0 + tid] = x;
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------- selection

// Keeps the first k_eff candidates by (score desc, index asc) and writes their
// ids ascending to out[0..k_eff); `sc` holds the n scores.
// Radix select reading the scores from shared memory in every pass, for
// more candidates than the register version holds (portable router only).
__device__ void select_emit_large(const float* sc, const Cands& cd, int k_eff, int32_t* out,
                            int* hist, int* tmp) {
  const int tid = threadIdx.x;
  const int n = cd.n;
  const bool take_all = k_eff >= n;
  uint32_t prefix = 0, pmask = 0;
  int k_rem = k_eff;
  __shared__ int s_digit, s_above;
  if (!take_all) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      hist[tid] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kRouteThreads) {
        const uint32_t key = score_key(sc[i]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
      }
      __syncthreads();
      // inclusive suffix sums: thread t covers digit 255 - t
      const int cnt = hist[255 - tid];
      int total;
      const int excl = block_excl_scan(cnt, tmp, &total);
      const int incl = excl + cnt;
      if (incl >= k_rem && excl < k_rem) {
        s_digit = 255 - tid;
        s_above = excl;
      }
      __syncthreads();
      prefix |= (uint32_t)s_digit << shift;
      pmask |= 255u << shift;
      k_rem -= s_above;
      __syncthreads();
    }
  }
  // ordered emission: thread t owns candidates [t*per, (t+1)*per)
  const int per = (n + kRouteThreads - 1) / kRouteThreads;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int n_eq = 0;
  if (!take_all)
    for (int i = i0; i < i1; ++i) n_eq += score_key(sc[i]) == prefix;
  int tot;
  int eq_before = block_excl_scan(n_eq, tmp, &tot);
  int n_keep = 0;
  for (int i = i0; i < i1; ++i) {
    bool keep = take_all;
    if (!take_all) {
      const uint32_t key = score_key(sc[i]);
      if (key > prefix) keep = true;
      else if (key == prefix) keep = (eq_before++) < k_rem;
    }
    n_keep += keep;
  }
  int pos = block_excl_scan(n_keep, tmp, &tot);
  eq_before -= n_eq;  // restore for the second walk
  for (int i = i0; i < i1; ++i) {
    bool keep = take_all;
    if (!take_all) {
      const uint32_t key = score_key(sc[i]);
      if (key > prefix) keep = true;
      else if (key == prefix) keep = (eq_before++) < k_rem;
    }
    if (keep && pos < k_eff) out[pos++] = cd.id(i);
  }
}

constexpr int kSelPer = 16;   // candidates per thread held in registers (n <= 4096)

__device__ void select_emit(const float* sc, const Cands& cd, int k_eff, int32_t* out,
                            int* hist, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int n = cd.n;
  if (k_eff >= n) {
    for (int i = tid; i < n; i += kRouteThreads) out[i] = cd.id(i);
    return;
  }
  // Thread t owns candidates [t*per, t*per + cnt) and keeps their keys in
  // registers for every pass (the selection is latency-bound: a dependent
  // shared-memory load, shuffle or barrier costs tens of cycles here).
  const int per = (n + kRouteThreads - 1) / kRouteThreads;
  if (per > kSelPer) {
    select_emit_large(sc, cd, k_eff, out, hist, tmp);
    return;
  }
  const int i0 = min(n, tid * per), cnt = min(n, i0 + per) - i0;
  uint32_t kr[kSelPer];
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) kr[e] = e < cnt ? score_key(sc[i0 + e]) : 0u;
  // ---- radix select of the k-th largest key, most significant bits first.
  // Bits every key shares (the scores of one block mostly agree in sign and
  // exponent) need no pass: the first pass starts at the highest bit where
  // the largest and smallest keys differ.  Each pass: one histogram of an
  // (up to) 8-bit digit, scanned by warp 0 alone; the histogram is double
  // buffered so a pass costs two barriers.
  __shared__ int s_digit, s_above, s_in_digit;
  __shared__ unsigned s_kmax, s_kmin;
  int* const hb1 = tmp + 32;                     // tmp holds 32 + 256 ints
  unsigned kmax = 0u, kmin = 0xffffffffu;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e)
    if (e < cnt) {
      kmax = max(kmax, kr[e]);
      kmin = min(kmin, kr[e]);
    }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  if (tid == 0) {
    s_kmax = 0u;
    s_kmin = 0xffffffffu;
  }
  hist[tid] = 0;
  hb1[tid] = 0;
  __syncthreads();
  if (lane == 0) {
    atomicMax(&s_kmax, kmax);
    atomicMin(&s_kmin, kmin);
  }
  __syncthreads();
  const uint32_t diff = s_kmax ^ s_kmin;
  int top = diff ? 31 - __clz(diff) : -1;          // highest differing bit
  uint32_t pmask = top < 0 ? 0xffffffffu : (top == 31 ? 0u : ~((2u << top) - 1u));
  uint32_t prefix = s_kmax & pmask;
  int k_rem = k_eff;
  // at most 4 passes (32 bits, <= 8 per pass); unrolled so that each pass's
  // histogram buffer is known at compile time
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    if (top < 0) break;
    int* const hcur = (pass & 1) ? hb1 : hist;
    int* const hnxt = (pass & 1) ? hist : hb1;
    const int shift = max(0, top - 7);
    const uint32_t dmask = (2u << (top - shift)) - 1u;   // digit of <= 8 bits
#pragma unroll
    for (int e = 0; e < kSelPer; ++e)
      if (e < cnt && (kr[e] & pmask) == prefix) atomicAdd(&hcur[(kr[e] >> shift) & dmask], 1);
    __syncthreads();
    if (w == 0) {
      // lane l covers digits 255-8l .. 248-8l (descending); find the digit
      // where the count of larger digits first reaches k_rem
      int c8[8], sum = 0;
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        c8[x] = hcur[255 - 8 * lane - x];
        sum += c8[x];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;                          // counts of larger digits
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        if (run < k_rem && run + c8[x] >= k_rem) {
          s_digit = 255 - 8 * lane - x;
          s_above = run;
          s_in_digit = c8[x];
        }
        run += c8[x];
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) hnxt[8 * lane + x] = 0;   // clear for the next pass
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    pmask |= dmask << shift;
    k_rem -= s_above;
    top = shift - 1;
    // every key that shares the resolved prefix is kept: the k-th key need
    // not be resolved further (the kept set is the same)
    if (s_in_digit == k_rem) break;
  }
  // ---- ordered emission.  One scan of packed counts (keys above the k-th
  // key, keys equal to it, both on the resolved bits pmask) gives every kept
  // candidate its slot: the larger keys before it plus the first k_rem equal
  // keys (by position).
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e)
    if (e < cnt) {
      n_gt += (kr[e] & pmask) > prefix;
      n_eq += (kr[e] & pmask) == prefix;
    }
  int tot;
  const int packed = block_excl_scan((n_gt << 16) | n_eq, tmp, &tot);
  int gt_before = packed >> 16, eq_before = packed & 0xffff;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    if (e >= cnt) break;
    const uint32_t km = kr[e] & pmask;
    if (km > prefix) {
      out[gt_before + min(eq_before, k_rem)] = cd.id(i0 + e);
      ++gt_before;
    } else if (km == prefix) {
      if (eq_before < k_rem) out[gt_before + eq_before] = cd.id(i0 + e);
      ++eq_before;
    }
  }
}

// Kept chunks of (b, h) from the chunk router's output, compacted into smem:
// entry i is kept when it lies in the candidate window [lo, hi) and exceeds
// entry i-1 (the list must be strictly ascending).  Anything else is reported
// (HGA_ERR_DEVICE_CHECK) and dropped.  All 256 threads load and test entries
// in parallel; returns the count.
__device__ int compact_kept_chunks(const RouteArgs& a, int b, int h, int lo, int64_t hi,
                                   int* kept, int* s_n, int* tmp) {
  const int32_t* in = a.in_idx + ((int64_t)h * a.n_blocks + b) * a.in_cap;
  // the first round's entries are read in the same round as the count (the
  // row holds in_cap slots, so these reads stay inside it whatever the count)
  const int lim = (int)min(a.in_cap, (int64_t)2048);
  const int c_first = threadIdx.x < lim ? in[threadIdx.x] : -1;
  const int p_first = threadIdx.x >= 1 && threadIdx.x - 1 < lim ? in[threadIdx.x - 1] : -1;
  int cnt = a.in_cnt[(int64_t)h * a.n_blocks + b];
  if (cnt < 0 || cnt > a.in_cap || cnt > 2048) {
    if (threadIdx.x == 0) report(HGA_ERR_DEVICE_CHECK);
    cnt = 0;
  }
  int base = 0;
  for (int i0 = 0; i0 < cnt; i0 += kRouteThreads) {
    const int i = i0 + threadIdx.x;
    int c = -1;
    bool ok = false;
    if (i < cnt) {
      c = i0 == 0 ? c_first : in[i];
      const int prev = i > 0 ? (i0 == 0 ? p_first : in[i - 1]) : -1;
      ok = c >= lo && c < hi && c > prev;
      if (!ok) report(HGA_ERR_DEVICE_CHECK);
    }
    int total;
    const int pos = block_excl_scan(ok ? 1 : 0, tmp, &total);
    if (ok) kept[base + pos] = c;
    base += total;
  }
  if (threadIdx.x == 0) *s_n = base;
  __syncthreads();
  return *s_n;
}

// ---------------------------------------------------------------- kernel

template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteArgs a) {
  extern __shared__ __align__(128) char smem[];
  griddep_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int64_t b0 = a.q_start + (int64_t)b * a.qblock;
  const int npos = (int)min((int64_t)a.qblock, a.q_start + a.n_q - b0);
  const int nrows = npos * a.G;
  __shared__ int s_kept[2048];
  __shared__ int s_nkept;
  __shared__ int hist[256];
  __shared__ int tmp[32 + 256];          // scan slots + second histogram buffer

  // ---- candidates
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
  if (k_eff > a.out_cap || cd.n > a.max_cands) {   // host sizing guarantees this
    if (threadIdx.x == 0) report(HGA_ERR_DEVICE_CHECK);
    return;
  }
  for (int i = k_eff + threadIdx.x; i < a.out_cap; i += kRouteThreads) out[i] = -1;
  if (threadIdx.x == 0) a.out_cnt[(int64_t)h * a.n_blocks + b] = k_eff;
  if (k_eff == 0) return;

  // ---- scores (skipped when every candidate is kept)
  float* sc = reinterpret_cast<float*>(smem);
  char* rest = smem + ((a.max_cands * 4 + 127) & ~127);
  if (k_eff < cd.n) {
    if constexpr (sizeof(T) == 2) {
      char* sq = rest;
      char* tiles = sq + kRouteMaxRowsBf16 * D * 2;
      float* red = reinterpret_cast<float*>(tiles + 2 * kRouteTile * D * 2);
      score_bf16<D>(a, b, h, (int)b0, nrows, cd, sc, sq, tiles, red);
    } else {
      float* sq = reinterpret_cast<float*>(rest);
      float* stile = sq + kRouteMaxRowsF32 * (D + 1);
      float* red = stile + kRouteTile * (D + 1);
      score_f32<D>(a, b, h, (int)b0, nrows, cd, sc, sq, stile, red);
    }
  }
  griddep_launch();
  select_emit(sc, cd, k_eff, out, hist, tmp);
}

template <typename T, int D>
inline size_t route_smem_bytes(int max_cands) {
  size_t s = ((size_t)max_cands * 4 + 127) & ~(size_t)127;
  if (sizeof(T) == 2)
    s += (size_t)kRouteMaxRowsBf16 * D * 2 + 2 * kRouteTile * D * 2 +
         (kRouteThreads / 32) * kRouteTile * 4;
  else
    s += ((size_t)kRouteMaxRowsF32 + kRouteTile) * (D + 1) * 4 +
         (kRouteThreads / kRouteTile) * kRouteTile * 4;
  return s;
}

}  // namespace hga
