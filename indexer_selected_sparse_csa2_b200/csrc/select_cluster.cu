// Exact Top-K of decode rows on thread-block clusters (lowest-position
// tie-break, ascending output).
//
// Selection rule of the lightning indexer (Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row: each query
// attends only to its index_topk best-scored tokens); the hierarchical pool
// of the DeepSeek-V4.1 blog (CSA2 paragraph) and of the architecture database
// ("2048-block x 8-position candidate pool") is the same selection over block
// maxima, expanded to the blocks' positions.
//
// One cluster of 8 CTAs (16 for rows over 2^16 slots) per (row, job).  Warp w
// of CTA c scans the run [(32c + w) * run, +run) of the row, 4 slots per lane
// per 128-slot step.
//   1. the first-level bin beta holding the K-th largest order key, and r,
//      the number still needed from that bin, from a 4096-bin histogram of
//      key >> 20: built by the producer of the values, or, in the fused pool
//      variant, here (CTA c owns bins [c*SEG, (c+1)*SEG) and receives the
//      others' counts through distributed shared memory; the owner holding
//      the crossing publishes beta);
//   2. every slot is classified against beta: slots of bin >= beta go to the
//      warp's list in slot order, keys of bin beta to a CTA list, sent to
//      CTA 0 in one batch;
//   3. CTA 0 runs two 10-bit radix passes over the gathered keys: the exact
//      K-th key tau and the number of slots equal to tau to take (lowest
//      slots first).  With more keys in bin beta than CTA 0 holds (heavy
//      ties) every CTA rescans its slots per pass and the digit counts are
//      summed in CTA 0 instead;
//   4. ordered emission: counts of keys equal to tau and of selected slots
//      are scanned over lanes (ballots), warps and the cluster's CTAs (their
//      totals read through distributed shared memory), and each selected
//      slot is written at its rank.
// Results one CTA computes for all (segment totals, beta, tau) are pushed
// into every CTA's shared memory before a cluster barrier, so no CTA reads a
// peer's shared memory late and no closing barrier is needed.
// Two pool variants take their values from the candidate pool instead of a
// row in memory: one scores its slice of the pool positions itself (gathered
// FP8 keys, mma.sync m16n8k32 e4m3, ReLU, head weights), the other gathers the
// scores a scorer already wrote; both keep the values in shared memory.
// Selecting inside the pool is exact for a pool-building call whenever the
// pool keeps at least K blocks: every one of the K best positions lies in
// one of the K best blocks (ranking blocks by max, then lower block; see
// run_index_decode).  No wait here is a spin: cluster barriers are hardware
// barriers that every thread of every CTA reaches the same number of times.
#include <algorithm>

#include "select.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kCsThreads = 1024;
constexpr int kCsWarps = kCsThreads / 32;
constexpr int kCsGatherCap = 8192;     // keys of bin beta gathered in CTA 0 (fast path)
constexpr int kCsWarpCap = 192;        // slots of bin >= beta listed per warp
constexpr int kCsBatch = 4;            // 128-slot steps whose loads are in flight together
constexpr int kCsSliceCap = 8192;      // pool variants: values per CTA in shared memory
constexpr int kCsLongRow = 1 << 16;    // rows above this use clusters of 16 CTAs, else 8
constexpr int kCsMaxCluster = 16;

enum CsMode : int { kCsRows = 0, kCsPoolScore = 1, kCsPoolGather = 2 };

struct CsSmem {
  uint32_t wl_key[kCsWarps][kCsWarpCap];          // per warp, slot order: keys of bin >= beta
  int32_t wl_slot[kCsWarps][kCsWarpCap];          // ... and their slots
  uint32_t gat_key[kCsGatherCap];                 // CTA 0: the keys of bin beta of the whole row
  uint32_t cand_key[kCsGatherCap];                // this CTA's keys of bin beta
  uint32_t h_loc[1024];
  uint32_t h_red[2][1024];                        // CTA 0: summed digit histograms (slow path)
  uint32_t warp_tot[2][kCsWarps];
  uint32_t tot_in[3][kCsMaxCluster];              // pushed by every CTA: segment, eq, selected totals
  uint32_t scan_tot;
  uint32_t gat_n;                                 // CTA 0: keys gathered
  uint32_t cand_n;                                // this CTA's keys of bin beta
  uint32_t gat_base;
  int beta;                                       // first-level bin of the K-th key
  uint32_t r_rem;                                 // keys still needed from bin beta
  uint32_t n_beta;                                // keys in bin beta (whole row)
  int take_all;
  uint32_t tau;                                   // the K-th key
  uint32_t need_eq;                               // keys equal to tau to take
  uint32_t all_eq;                                // every key equal to tau is taken
  uint32_t digit;
  uint32_t dcount;                                // keys in the found digit
  int owner;
  int last_selected;
  float sv[kCsSliceCap];                          // pool variants
  uint32_t hist_loc[kHistBins];
  uint32_t hist_red[kHistBins];                   // owner CTAs: the merged 4096-bin histogram
};

// Inclusive scan over the 1024 threads; *total gets the sum.  Ends with a
// barrier, so the scratch may be reused right away.
CSA_DEV uint32_t cs_block_scan(uint32_t v, uint32_t* wtot, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) wtot[wid] = v;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = wtot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    wtot[lane] = w;
    if (lane == 31) *total = w;
  }
  __syncthreads();
  const uint32_t r = v + (wid > 0 ? wtot[wid - 1] : 0u);
  __syncthreads();
  return r;
}

// Exclusive scan of the 32 per-warp counts in wt (in place) by warp 0; returns
// the CTA total to every thread.  Called by all threads.
CSA_DEV uint32_t cs_warp_counts_scan(uint32_t* wt, uint32_t* total) {
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const uint32_t v = wt[lane];
    uint32_t s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    wt[lane] = s - v;
    if (lane == 31) *total = s;
  }
  __syncthreads();
  return *total;
}

// Radix digit search over 1024 counts held one per thread, for digit
// 1023 - tid (so the scan walks the digits from the top down): the digit
// holding the r-th largest key, how many keys of it are still needed and how
// many it holds.  Called by all threads; results in S.digit / S.need_eq /
// S.dcount.
CSA_DEV void cs_find_digit(CsSmem& S, uint32_t count, uint32_t r) {
  const uint32_t incl = cs_block_scan(count, S.warp_tot[0], &S.scan_tot);
  if (incl - count < r && incl >= r) {
    S.digit = 1023u - threadIdx.x;
    S.need_eq = r - (incl - count);
    S.dcount = count;
  }
  __syncthreads();
}

CSA_DEV void cs_write(const CsRow& J, int b, uint32_t j, int64_t slot) {
  int32_t* out = J.out + (int64_t)b * J.out_stride;
  const int32_t pos = J.map ? J.map[(int64_t)b * J.map_stride + slot] : (int32_t)slot;
  if (J.expand == 0) {
    out[j] = pos;
  } else {
    for (int r = 0; r < J.expand; ++r) {
      const int64_t p = (int64_t)pos * J.expand + r;
      out[(int64_t)j * J.expand + r] = p < J.limit ? (int32_t)p : -1;
    }
  }
}

CSA_DEV void mma_e4m3_16832_cs(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MODE, int CL>
__global__ void __launch_bounds__(kCsThreads, 1) cluster_select_kernel(CsJobs jobs, CsPool pp) {
  constexpr bool POOL = MODE != kCsRows;
  // shared-memory setup and the cluster's first arrival overlap the previous
  // kernel; every global read comes after the wait below
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t cs_raw[];
  CsSmem& S = *reinterpret_cast<CsSmem*>(cs_raw);
  const CsRow& J = jobs.j[blockIdx.z];
  const int b = blockIdx.y;
  const uint32_t rank = cluster_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const uint32_t K = (uint32_t)J.K;

  for (int i = tid; i < 1024; i += kCsThreads) { S.h_red[0][i] = 0; S.h_red[1][i] = 0; }
  if (POOL)
    for (int i = tid; i < kHistBins; i += kCsThreads) { S.hist_loc[i] = 0; S.hist_red[i] = 0; }
  if (tid == 0) {
    S.gat_n = 0; S.cand_n = 0; S.last_selected = 0; S.beta = 0; S.r_rem = 0; S.n_beta = 0;
    S.take_all = 0; S.all_eq = 0; S.tau = 0; S.need_eq = 0;
  }
  __syncthreads();
  // peers write into this CTA's shared memory only after the matching wait
  cluster_arrive();
  pdl_wait();

  const int64_t nrow = POOL ? min((int64_t)pp.pool_len[b], J.n) : (J.n_row ? min((int64_t)J.n_row[b], J.n) : J.n);
  const int64_t run = J.run;
  const int64_t cta_lo = (int64_t)rank * kCsWarps * run;
  const int64_t lo_w = cta_lo + (int64_t)warp * run;
  const int64_t hi_w = max(lo_w, min(lo_w + run, nrow));
  const int steps = (int)((hi_w - lo_w + 127) / 128);
  const float* vrow = POOL ? nullptr : J.vals + (int64_t)b * J.row_stride;

  if (POOL) {
    const int64_t chi = min(cta_lo + kCsWarps * run, nrow);
    const int32_t* pl = J.map + (int64_t)b * J.map_stride;
    if (MODE == kCsPoolScore) {
      // ----------------------------------------------- fused scores
      // slots [cta_lo, chi) of the pool in 16-slot tiles; lane (g, t) loads key
      // bytes [16t, 16t + 16) of tile rows g and g + 8
      const int g = lane >> 2, t = lane & 3;
      uint32_t qf[4] = {0u, 0u, 0u, 0u};
      if (g < pp.H_I) {
        const uint4 v = ld_v4(pp.q + ((int64_t)b * pp.H_I + g) * kDI + 16 * t);
        qf[0] = v.x; qf[1] = v.y; qf[2] = v.z; qf[3] = v.w;
      }
      const float w0 = (2 * t < pp.H_I) ? pp.w[(int64_t)b * pp.H_I + 2 * t] : 0.f;
      const float w1 = (2 * t + 1 < pp.H_I) ? pp.w[(int64_t)b * pp.H_I + 2 * t + 1] : 0.f;
      const uint8_t* kb = pp.keys + (int64_t)b * pp.key_batch_stride;
      const int ntile = (int)((chi - cta_lo + 15) / 16);
      constexpr int kTPW = 4;                     // tiles per warp per round (loads in flight)
      for (int t0 = warp; t0 < max(ntile, 0); t0 += kCsWarps * kTPW) {
        int32_t ps[kTPW][2];
#pragma unroll
        for (int u = 0; u < kTPW; ++u) {
          const int64_t r0 = cta_lo + 16 * (int64_t)(t0 + u * kCsWarps) + g;
          ps[u][0] = r0 < chi ? pl[r0] : -1;
          ps[u][1] = r0 + 8 < chi ? pl[r0 + 8] : -1;
        }
        uint4 ka[kTPW], kc[kTPW];
#pragma unroll
        for (int u = 0; u < kTPW; ++u) {
          ka[u] = ps[u][0] >= 0 ? ld_nc_v4(kb + (int64_t)ps[u][0] * pp.key_row_stride + 16 * t) : make_uint4(0, 0, 0, 0);
          kc[u] = ps[u][1] >= 0 ? ld_nc_v4(kb + (int64_t)ps[u][1] * pp.key_row_stride + 16 * t) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kTPW; ++u) {
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          mma_e4m3_16832_cs(c, ka[u].x, kc[u].x, ka[u].y, kc[u].y, qf[0], qf[1]);
          mma_e4m3_16832_cs(c, ka[u].z, kc[u].z, ka[u].w, kc[u].w, qf[2], qf[3]);
          float s_lo = w0 * fmaxf(c[0], 0.f) + w1 * fmaxf(c[1], 0.f);
          float s_hi = w0 * fmaxf(c[2], 0.f) + w1 * fmaxf(c[3], 0.f);
          s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
          s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
          s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
          s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
          const int64_t r0 = cta_lo + 16 * (int64_t)(t0 + u * kCsWarps) + g;
          const int64_t r = t == 0 ? r0 : r0 + 8;
          const float sc = t == 0 ? s_lo : s_hi;
          if (t < 2 && r < chi) {
            S.sv[r - cta_lo] = sc;
            if (pp.scores) pp.scores[(int64_t)b * J.row_stride + r] = sc;
            atomicAdd(&S.hist_loc[order_key(sc) >> (32 - kHistBits)], 1u);
          }
        }
      }
    } else {
      // ------------------------------------- scores gathered by pool position
      constexpr int kG = kCsSliceCap / kCsThreads;
      const float* gs = pp.gscores + (int64_t)b * pp.gscore_stride;
      int32_t ps[kG];
#pragma unroll
      for (int u = 0; u < kG; ++u) {
        const int64_t r = cta_lo + tid + (int64_t)u * kCsThreads;
        ps[u] = r < chi ? pl[r] : -1;
      }
      float v[kG];
#pragma unroll
      for (int u = 0; u < kG; ++u) v[u] = ps[u] >= 0 ? gs[ps[u]] : 0.f;
#pragma unroll
      for (int u = 0; u < kG; ++u) {
        const int64_t r = cta_lo + tid + (int64_t)u * kCsThreads;
        if (r < chi) {
          S.sv[r - cta_lo] = v[u];
          atomicAdd(&S.hist_loc[order_key(v[u]) >> (32 - kHistBits)], 1u);
        }
      }
    }
    __syncthreads();
    // ---- 1. merge the 4096-bin histogram: CTA c owns bins [c*SEG, (c+1)*SEG)
    constexpr int SEG = kHistBins / CL;
    cluster_wait();                                   // the owners' bins are cleared
    for (int i = tid; i < kHistBins; i += kCsThreads) {
      const uint32_t v = S.hist_loc[i];
      if (v) dsmem_add(dsmem(&S.hist_red[i], (uint32_t)(i / SEG)), v);
    }
    cluster_sync_all();
    {
      const uint32_t v = tid < SEG ? S.hist_red[rank * SEG + tid] : 0u;
      cs_block_scan(v, S.warp_tot[0], &S.scan_tot);
      if (tid < CL) dsmem_st(dsmem(&S.tot_in[0][rank], (uint32_t)tid), S.scan_tot);
    }
    cluster_sync_all();
    // owner totals from the top segment down: the crossing owner and the
    // count above its segment
    if (warp == 0) {
      const uint32_t c = lane < CL ? S.tot_in[0][CL - 1 - lane] : 0u;
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t2 = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t2;
      }
      const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) { S.take_all = total <= K; S.owner = 0; }
      __syncwarp();
      if (total > K && incl - c < K && incl >= K) { S.owner = CL - 1 - lane; S.r_rem = K - (incl - c); }
    }
    __syncthreads();
    const bool take_all_p = S.take_all != 0;
    if (!take_all_p && (int)rank == S.owner) {
      // the owner walks its segment from the top bin down and pushes beta
      const int bin = (int)rank * SEG + SEG - 1 - tid;
      const uint32_t c = tid < SEG ? S.hist_red[bin] : 0u;
      const uint32_t r = S.r_rem;
      const uint32_t incl = cs_block_scan(c, S.warp_tot[0], &S.scan_tot);
      if (tid < SEG && incl - c < r && incl >= r) {
        for (int d = 0; d < CL; ++d) {
          dsmem_st(dsmem(&S.beta, (uint32_t)d), (uint32_t)bin);
          dsmem_st(dsmem(&S.r_rem, (uint32_t)d), r - (incl - c));
          dsmem_st(dsmem(&S.n_beta, (uint32_t)d), c);
        }
      }
    }
    cluster_sync_all();
  } else {
    // ---- 1. first-level bin beta from the row's 4096-bin histogram
    // thread i holds bins [4(1023 - i), +4): scanning threads in order walks
    // the bins from the top down
    const int base = 4 * (1023 - tid);
    uint32_t h4[4], sum = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h4[k] = J.hist[(int64_t)b * kHistBins + base + k];
      sum += h4[k];
    }
    const uint32_t incl = cs_block_scan(sum, S.warp_tot[0], &S.scan_tot);
    const uint32_t excl = incl - sum;
    if (tid == 0) S.take_all = S.scan_tot <= K;
    __syncthreads();
    if (!S.take_all && excl < K && incl >= K) {
      uint32_t cum = excl;
      for (int k = 3; k >= 0; --k) {
        if (cum + h4[k] >= K) { S.beta = base + k; S.r_rem = K - cum; S.n_beta = h4[k]; break; }
        cum += h4[k];
      }
    }
    __syncthreads();
    cluster_wait();                                   // CTA 0's gather buffer is ready
  }
  const bool take_all = S.take_all != 0;
  const uint32_t beta_key = (uint32_t)S.beta << 20;   // keys >= this are in bins >= beta
  // the keys of bin beta fit CTA 0's buffer: gather them there
  const bool gather = !take_all && S.n_beta <= (uint32_t)kCsGatherCap;

  auto load4 = [&](int64_t s0, float (&x)[4]) -> uint32_t {
    uint32_t valid = 0;
    if (POOL) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[j] = s0 + j < hi_w ? S.sv[s0 + j - cta_lo] : 0.f;
        valid |= (s0 + j < hi_w ? 1u : 0u) << j;
      }
    } else if (s0 + 3 < hi_w && J.vec) {
      const float4 f = *reinterpret_cast<const float4*>(vrow + s0);
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      valid = 0xFu;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[j] = s0 + j < hi_w ? vrow[s0 + j] : 0.f;
        valid |= (s0 + j < hi_w ? 1u : 0u) << j;
      }
    }
    return valid;
  };

  // ------------------------------------------- 2. classify, list, collect bin beta
  // Slots of bin >= beta go to the warp's list in slot order; with `gather`,
  // keys of bin beta also to the CTA's list (any order).
  uint32_t wcnt = 0;                                  // warp-uniform
  for (int k0 = 0; k0 < steps; k0 += kCsBatch) {
    float x[kCsBatch][4];
    uint32_t valid[kCsBatch];
#pragma unroll
    for (int u = 0; u < kCsBatch; ++u)
      valid[u] = k0 + u < steps ? load4(lo_w + 128 * (int64_t)(k0 + u) + 4 * lane, x[u]) : 0u;
#pragma unroll
    for (int u = 0; u < kCsBatch; ++u) {
      uint32_t key[4], ge = 0, cb = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        key[j] = order_key(x[u][j]);
        if ((valid[u] >> j) & 1u) {
          if (take_all || key[j] >= beta_key) ge |= 1u << j;
          if (gather && (key[j] >> 20) == (beta_key >> 20)) cb |= 1u << j;
        }
      }
      if (__any_sync(0xffffffffu, ge != 0)) {
        const uint32_t n = __popc(ge);
        uint32_t pre = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, pre, o);
          if (lane >= o) pre += t;
        }
        uint32_t at = wcnt + pre - n;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((ge >> j) & 1u) {
            if (at < (uint32_t)kCsWarpCap) {
              S.wl_key[warp][at] = key[j];
              S.wl_slot[warp][at] = (int32_t)(lo_w + 128 * (int64_t)(k0 + u) + 4 * lane + j);
            }
            ++at;
          }
        wcnt += __shfl_sync(0xffffffffu, pre, 31);
      }
      if (gather && __any_sync(0xffffffffu, cb != 0)) {
        const uint32_t n = __popc(cb);
        uint32_t pre = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, pre, o);
          if (lane >= o) pre += t;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, pre, 31);
        uint32_t at = 0;
        if (lane == 31) at = atomicAdd(&S.cand_n, tot);
        at = __shfl_sync(0xffffffffu, at, 31) + pre - n;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((cb >> j) & 1u) S.cand_key[at++] = key[j];   // < n_beta <= kCsGatherCap
      }
    }
  }
  const bool wfast = wcnt <= (uint32_t)kCsWarpCap;  // else this warp re-reads its run
  __syncthreads();

  // ------------------------------------------- 3. exact tau by two radix passes
  if (!take_all) {
    uint32_t prefix = beta_key >> 20, r = S.r_rem;
    if (gather) {
      // this CTA's keys of bin beta to CTA 0, in one batch
      const uint32_t n_mine = S.cand_n;
      if (tid == 0) S.gat_base = n_mine ? dsmem_atom_add(dsmem(&S.gat_n, 0), n_mine) : 0u;
      __syncthreads();
      const uint32_t base = S.gat_base;
      for (uint32_t i = tid; i < n_mine; i += kCsThreads) dsmem_st(dsmem(&S.gat_key[base + i], 0), S.cand_key[i]);
      cluster_sync_all();                             // every key of bin beta is in CTA 0
      if (rank == 0) {
        const uint32_t n = S.gat_n;
        for (int pass = 0; pass < 2; ++pass) {
          const int shift = pass == 0 ? 10 : 0;       // digit bits 19..10, then 9..0
          S.h_loc[tid] = 0u;
          __syncthreads();
          for (uint32_t i = tid; i < n; i += kCsThreads) {
            const uint32_t key = S.gat_key[i];
            if ((key >> (shift + 10)) == prefix) atomicAdd(&S.h_loc[(key >> shift) & 1023u], 1u);
          }
          __syncthreads();
          cs_find_digit(S, S.h_loc[1023 - tid], r);
          prefix = (prefix << 10) | S.digit;
          r = S.need_eq;
          __syncthreads();
        }
        // push tau to every CTA
        if (tid < CL) {
          dsmem_st(dsmem(&S.tau, (uint32_t)tid), prefix);
          dsmem_st(dsmem(&S.need_eq, (uint32_t)tid), r);
          dsmem_st(dsmem(&S.all_eq, (uint32_t)tid), r == S.dcount ? 1u : 0u);
        }
      }
      cluster_sync_all();                             // tau is everywhere
    } else {
      // more keys in bin beta than CTA 0 holds (heavy ties): each pass rescans
      // the warps' runs and sums digit histograms in CTA 0
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        S.h_loc[tid] = 0u;
        __syncthreads();
        for (int k = 0; k < steps; ++k) {
          float x[4];
          const uint32_t valid = load4(lo_w + 128 * (int64_t)k + 4 * lane, x);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t key = order_key(x[j]);
            if (((valid >> j) & 1u) && (key >> (shift + 10)) == prefix)
              atomicAdd(&S.h_loc[(key >> shift) & 1023u], 1u);
          }
        }
        __syncthreads();
        const uint32_t v = S.h_loc[tid];
        if (v) dsmem_add(dsmem(&S.h_red[pass][tid], 0), v);
        cluster_sync_all();
        cs_find_digit(S, dsmem_ld(dsmem(&S.h_red[pass][1023 - tid], 0)), r);
        prefix = (prefix << 10) | S.digit;
        r = S.need_eq;
        __syncthreads();
      }
      if (tid == 0) { S.tau = prefix; S.need_eq = r; S.all_eq = r == S.dcount ? 1u : 0u; }
      __syncthreads();
    }
  }
  const uint32_t tau = S.tau;
  const uint32_t need_eq = S.need_eq;
  // ranks among keys equal to tau matter only when some of them are left out
  const bool ranks = !take_all && S.all_eq == 0;

  // ------------------------------------------- 4. ordered emission
  // A warp whose list overflowed walks its run again from the values
  // (4 slots per lane per step, ranks by ballots); otherwise it walks its
  // list, 32 entries at a time.
  const uint32_t nl = min(wcnt, (uint32_t)kCsWarpCap);
  auto step_ge = [&](int k, uint32_t (&key)[4]) -> uint32_t {
    float x[4];
    const uint32_t valid = load4(lo_w + 128 * (int64_t)k + 4 * lane, x);
    uint32_t ge = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      key[j] = order_key(x[j]);
      if (((valid >> j) & 1u) && (take_all || key[j] >= beta_key)) ge |= 1u << j;
    }
    return ge;
  };
  // a. keys equal to tau per warp, ranked across the cluster
  uint32_t eq_base = 0;
  if (ranks) {
    uint32_t n_eq = 0;
    if (wfast) {
      for (uint32_t e = lane; e < nl; e += 32) n_eq += S.wl_key[warp][e] == tau ? 1u : 0u;
    } else {
      for (int k = 0; k < steps; ++k) {
        uint32_t key[4];
        const uint32_t ge = step_ge(k, key);
#pragma unroll
        for (int j = 0; j < 4; ++j) n_eq += ((ge >> j) & 1u) && key[j] == tau ? 1u : 0u;
      }
    }
    n_eq = __reduce_add_sync(0xffffffffu, n_eq);
    if (lane == 0) S.warp_tot[0][warp] = n_eq;
    const uint32_t cta_eq = cs_warp_counts_scan(S.warp_tot[0], &S.scan_tot);
    if (tid < CL) dsmem_st(dsmem(&S.tot_in[1][rank], (uint32_t)tid), cta_eq);
    cluster_sync_all();
    uint32_t v = tid < (int)rank ? S.tot_in[1][tid] : 0u;
    v = __reduce_add_sync(0xffffffffu, tid < 32 ? v : 0u);
    if (tid == 0) S.scan_tot = v;
    __syncthreads();
    eq_base = S.scan_tot + S.warp_tot[0][warp];
    __syncthreads();
  }

  // selected among 32 list entries (or one step's 4 slots per lane), given the
  // rank of the chunk's first equal key; eq_run advances past its equal keys
  auto sel_list = [&](uint32_t e, uint32_t& eq_run) -> bool {
    const bool in = e < nl;
    const uint32_t key = in ? S.wl_key[warp][e] : 0u;
    if (take_all) return in;
    if (!ranks) return in && key >= tau;
    const bool eq = in && key == tau;
    const uint32_t bal = __ballot_sync(0xffffffffu, eq);
    const bool sel = in && (key > tau || (eq && eq_run + __popc(bal & lt) < need_eq));
    eq_run += __popc(bal);
    return sel;
  };
  auto sel_step = [&](int k, uint32_t& eq_run) -> uint32_t {
    uint32_t key[4];
    const uint32_t ge = step_ge(k, key);
    if (take_all) return ge;
    uint32_t eqb = 0, gtb = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if ((ge >> j) & 1u) {
        if (key[j] == tau) eqb |= 1u << j;
        else if (key[j] > tau) gtb |= 1u << j;
      }
    if (!ranks) return gtb | eqb;
    uint32_t before = 0, step_tot = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t bal = __ballot_sync(0xffffffffu, (eqb >> j) & 1u);
      before += __popc(bal & lt);
      step_tot += __popc(bal);
    }
    uint32_t sel = gtb;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if ((eqb >> j) & 1u) {
        if (eq_run + before < need_eq) sel |= 1u << j;
        ++before;
      }
    eq_run += step_tot;
    return sel;
  };

  // b. selected slots per warp, ranked across the cluster
  uint32_t n_sel = 0;
  {
    uint32_t eq_run = eq_base;
    if (wfast) {
      for (uint32_t e0 = 0; e0 < nl; e0 += 32) n_sel += sel_list(e0 + lane, eq_run) ? 1u : 0u;
    } else {
      for (int k = 0; k < steps; ++k) n_sel += __popc(sel_step(k, eq_run));
    }
  }
  n_sel = __reduce_add_sync(0xffffffffu, n_sel);
  if (lane == 0) S.warp_tot[1][warp] = n_sel;
  const uint32_t cta_sel = cs_warp_counts_scan(S.warp_tot[1], &S.scan_tot);
  if (tid < CL) dsmem_st(dsmem(&S.tot_in[2][rank], (uint32_t)tid), cta_sel);
  cluster_sync_all();
  uint32_t sel_base = 0, all_sel = 0;
  if (tid < CL) {
    const uint32_t v = S.tot_in[2][tid];
    sel_base = tid < (int)rank ? v : 0u;
    all_sel = v;
  }
  sel_base = __reduce_add_sync(0xffffffffu, tid < 32 ? sel_base : 0u);
  all_sel = __reduce_add_sync(0xffffffffu, tid < 32 ? all_sel : 0u);
  if (tid == 0) { S.scan_tot = sel_base; S.gat_base = all_sel; }
  __syncthreads();
  uint32_t out_at = S.scan_tot + S.warp_tot[1][warp];
  const uint32_t total = S.gat_base;

  // c. writes, in slot order
  {
    uint32_t eq_run = eq_base;
    if (wfast) {
      for (uint32_t e0 = 0; e0 < nl; e0 += 32) {
        const uint32_t e = e0 + lane;
        const bool sel = sel_list(e, eq_run);
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const int64_t slot = S.wl_slot[warp][e];
          cs_write(J, b, out_at + __popc(bal & lt), slot);
          if (slot == nrow - 1) S.last_selected = 1;
        }
        out_at += __popc(bal);
      }
    } else {
      for (int k = 0; k < steps; ++k) {
        const uint32_t sel = sel_step(k, eq_run);
        uint32_t before = 0, step_tot = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t bal = __ballot_sync(0xffffffffu, (sel >> j) & 1u);
          before += __popc(bal & lt);
          step_tot += __popc(bal);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((sel >> j) & 1u) {
            const int64_t slot = lo_w + 128 * (int64_t)k + 4 * lane + j;
            cs_write(J, b, out_at + before, slot);
            if (slot == nrow - 1) S.last_selected = 1;
            ++before;
          }
        out_at += step_tot;
      }
    }
  }

  // padding (spread over the cluster) and the valid length of an expanded row
  const int64_t E = J.expand ? J.expand : 1;
  int32_t* orow = J.out + (int64_t)b * J.out_stride;
  for (int64_t j = (int64_t)total * E + (int64_t)rank * kCsThreads + tid; j < J.out_width;
       j += (int64_t)CL * kCsThreads)
    orow[j] = -1;
  if (J.expand && J.out_len) {
    __syncthreads();
    const int64_t owner = nrow > 0 ? (nrow - 1) / (kCsWarps * run) : 0;
    if (tid == 0 && (int64_t)rank == owner) {
      const int64_t over = S.last_selected ? max((int64_t)0, nrow * J.expand - J.limit) : 0;
      J.out_len[b] = (int32_t)((int64_t)total * J.expand - over);
    }
  }
  // every access to a peer's shared memory happened before the last cluster
  // barrier: the CTA may leave
}

// ----------------------------------------------------------------- host --
static int cs_cluster(int64_t n) { return n > kCsLongRow ? 16 : 8; }

int64_t cs_run(int64_t n) {
  const int64_t ctas = cs_cluster(n);
  int64_t run = (n + ctas * kCsWarps - 1) / (ctas * kCsWarps);
  run = (run + 3) / 4 * 4;
  return run < 4 ? 4 : run;
}

bool cs_pool_ok(int64_t pool_cap) { return pool_cap <= kCsLongRow && kCsWarps * cs_run(pool_cap) <= kCsSliceCap; }

template <int MODE, int CL>
static cudaError_t launch_cs(const CsJobs& js, int njobs, int B, const CsPool& pp, cudaStream_t stream,
                             const char* name) {
  static SmemAttrOnce attr;
  cudaError_t e = attr.set(cluster_select_kernel<MODE, CL>, sizeof(CsSmem));
  if (e != cudaSuccess) return e;
  if (CL > 8) {
    static SmemAttrOnce np;   // once per device as well
    e = np.set_attr(cluster_select_kernel<MODE, CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, B, njobs);
  cfg.blockDim = dim3(kCsThreads);
  cfg.dynamicSmemBytes = sizeof(CsSmem);
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = CL;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  ProfScope ps(stream, name);
  e = cudaLaunchKernelEx(&cfg, cluster_select_kernel<MODE, CL>, js, pp);
  note_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Rows of one launch share a cluster size: the longest row decides it.
cudaError_t launch_cluster_select(const CsRow* rows, int njobs, int B, cudaStream_t stream, const char* name) {
  CsJobs js;
  js.j[0] = rows[0];
  js.j[1] = njobs > 1 ? rows[1] : rows[0];
  const int64_t n = njobs > 1 ? std::max(rows[0].n, rows[1].n) : rows[0].n;
  for (int i = 0; i < 2; ++i) js.j[i].run = cs_run(n);
  CsPool pp{};
  return cs_cluster(n) == 16 ? launch_cs<kCsRows, 16>(js, njobs, B, pp, stream, name)
                             : launch_cs<kCsRows, 8>(js, njobs, B, pp, stream, name);
}

cudaError_t launch_cluster_pool_select(const CsRow& row, const CsPool& pp, int B, cudaStream_t stream) {
  CsJobs js;
  js.j[0] = row;
  js.j[0].run = cs_run(row.n);
  js.j[1] = js.j[0];
  if (pp.gscores) return launch_cs<kCsPoolGather, 8>(js, 1, B, pp, stream, "pool_gather_select");
  return launch_cs<kCsPoolScore, 8>(js, 1, B, pp, stream, "pool_score_select");
}

}  // namespace csa
