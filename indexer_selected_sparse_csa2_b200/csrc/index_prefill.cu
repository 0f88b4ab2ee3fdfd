// Prefill indexer scoring + exact per-query Top-K for a chunk of n_q causal
// query tokens (lightning-indexer score S[t, s] = sum_j w[t,j] *
// relu(<qI[t,j], kI[s]>), s <= T - n_q + t; Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row).
//
// Dense part on the tensor cores: for a block of 24 queries (N = 24 x 8
// heads = 192 rows of 64 bytes) and 128-position key tiles (M = 128, TMA,
// 64-byte swizzle), two tcgen05.mma kind::f8f6f4 per tile into a 192-column
// TMEM accumulator (two of them, double-buffered).  Twelve epilogue warps
// (4 TMEM lane quarters x 3 groups of 8 queries) turn the head dots into
// scores.  The 1M x 4096 score
// matrix is never stored; selection is exact in three steps:
//   1  sample pass: the same kernel on every kSampleStride-th key tile writes
//      those scores; a Top-r select per query gives a threshold tau_t (the
//      r-th best sampled score), chosen so that ~2K positions should pass;
//   2  main pass: every (t, s) with S >= tau_t is appended (order key,
//      position) to query t's candidate region for that key chunk; each
//      (query block, key chunk) belongs to one CTA, so the append cursor is a
//      shared-memory counter (no global atomic round trip per hit);
//   3  final: per query, if its candidates provably contain the Top-K (at
//      least K of them, or tau = -inf, and no overflow) an exact radix select
//      with lowest-position tie-break runs on them; otherwise an exact
//      streaming fallback recomputes that query's scores on the CUDA cores.
#include "sm100.cuh"
#include "select.cuh"

namespace csa {

constexpr int kPfQPerBlock = 24;                      // queries per N block
constexpr int kPfN = kPfQPerBlock * 8;                // 192 (8 head rows per query)
constexpr int kPfRows = 128;
constexpr int kPfStages = 8;
constexpr int kPfStageBytes = kPfRows * 64;
constexpr int kPfAcc = 2;
constexpr int kPfEpiWarps = 12;                       // 4 TMEM quarters x 3 query groups of 8
constexpr int kPfThreads = 64 + 32 * kPfEpiWarps;     // 448 (register cap 128 per thread)
constexpr int kSampleStride = 64;                     // sample every 64th key tile
constexpr int kCandCap = 16384;                       // candidates the final select holds per query
constexpr int kChunkCapMax = 8192;                    // candidates kept per (query, key chunk), upper bound
constexpr int kPfChunkTiles = 256;                    // key tiles per work item

static __device__ int g_pf_error;

struct PfParams {
  const uint8_t* q;        // [B][n_q][H_I][64]
  const float* w;          // [B][n_q][H_I]
  int B, n_q, H_I;
  int64_t T;               // cache length; query t sits at T - n_q + t
  int mode;                // 0 = sample, 1 = main
  int n_items;             // work items (b, query block, key chunk)
  int qblocks;             // query blocks per sequence
  int kchunks;             // key chunks per query block
  int64_t ntiles;          // key tiles per sequence
  float* sample;           // [B*n_q][n_samp]    (mode 0)
  int64_t n_samp;
  const float* tau;        // [B*n_q]           (mode 1)
  uint2* cand;             // [B*n_q][kchunks][chunk_cap] (mode 1): (order key, position)
  int chunk_cap;
  uint32_t* cnt;           // [B*n_q][kchunks] hits per (query, key chunk), overflow included
};

struct PfSmem {
  uint8_t* stage;
  uint8_t* qb;             // 256 rows x 64 B (16 KB), 64-byte swizzle
  float* wts;              // [32 queries][8 heads] weights of the current block
  uint64_t* full;
  uint64_t* empty;
  uint64_t* accf;
  uint64_t* acce;
  uint32_t* tmem_base;
};

// 1 CTA per SM (the kernel takes all 512 TMEM columns): ask for > half the
// shared memory of an SM.
constexpr size_t kPfSmemBytes = 120 * 1024;

CSA_DEV PfSmem carve_pf_smem(uint8_t* raw) {
  PfSmem s;
  uintptr_t base = (reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  s.stage = p; p += (size_t)kPfStages * kPfStageBytes;
  s.qb = p; p += (size_t)kPfN * 64;
  s.wts = reinterpret_cast<float*>(p); p += kPfQPerBlock * 8 * 4;
  s.full = reinterpret_cast<uint64_t*>(p); p += kPfStages * 8;
  s.empty = reinterpret_cast<uint64_t*>(p); p += kPfStages * 8;
  s.accf = reinterpret_cast<uint64_t*>(p); p += kPfAcc * 8;
  s.acce = reinterpret_cast<uint64_t*>(p); p += kPfAcc * 8;
  s.tmem_base = reinterpret_cast<uint32_t*>(p);
  return s;
}

struct PfItem {
  int b, qb;
  int64_t kt0, kt1;        // key tile range (before sampling / causal trimming)
};

CSA_DEV PfItem pf_item(const PfParams& p, int it) {
  PfItem x;
  const int per_b = p.qblocks * p.kchunks;
  x.b = it / per_b;
  const int r = it - x.b * per_b;
  x.qb = r / p.kchunks;
  const int kc = r - x.qb * p.kchunks;
  x.kt0 = (int64_t)kc * kPfChunkTiles;
  x.kt1 = min(x.kt0 + kPfChunkTiles, p.ntiles);
  // causal (main pass only): no query of this block sees positions past its
  // last query; the sample pass visits every sampled tile and writes -inf for
  // invisible positions, so every sample column is written
  if (p.mode == 1) {
    const int64_t last_q = min((int64_t)(x.qb + 1) * kPfQPerBlock, (int64_t)p.n_q) - 1;
    const int64_t max_pos = p.T - p.n_q + last_q;
    x.kt1 = min(x.kt1, max_pos / kPfRows + 1);
  }
  return x;
}

// Number of tiles of the item that this mode visits, and the i-th of them.
CSA_DEV int64_t pf_count(const PfParams& p, const PfItem& x) {
  if (x.kt1 <= x.kt0) return 0;
  if (p.mode == 1) return x.kt1 - x.kt0;
  // sample mode: tiles with index % kSampleStride == 0
  const int64_t first = (x.kt0 + kSampleStride - 1) / kSampleStride * kSampleStride;
  return first < x.kt1 ? (x.kt1 - 1 - first) / kSampleStride + 1 : 0;
}
CSA_DEV int64_t pf_tile(const PfParams& p, const PfItem& x, int64_t i) {
  if (p.mode == 1) return x.kt0 + i;
  const int64_t first = (x.kt0 + kSampleStride - 1) / kSampleStride * kSampleStride;
  return first + i * kSampleStride;
}

// Twice the ReLU of two head dots, x + |x| (exact: 2x for x > 0, +0
// otherwise), as one packed fp32x2 add on the FMA pipe; the head weights are
// halved to match, so w * relu(x) = (w / 2) * (x + |x|) is the same product
// and every fused multiply-add rounds as with max(x, 0).
CSA_DEV float2 relu2(uint32_t a, uint32_t b) {
  const float2 x = make_float2(__uint_as_float(a), __uint_as_float(b));
  return __fadd2_rn(x, make_float2(fabsf(x.x), fabsf(x.y)));
}

template <int MODE>   // 0 = sample pass, 1 = main pass (p.mode must match)
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, PfParams p) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  PfSmem S = carve_pf_smem(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kPfStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < kPfAcc; ++i) { mbar_init(&S.accf[i], 1); mbar_init(&S.acce[i], kPfEpiWarps); }
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  if (warp == 1) tmem_alloc(S.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *S.tmem_base;

  // running tile counter across items keeps the barrier phases consistent
  int64_t run = 0;
  int64_t issued = 0;                  // key-tile copies issued (producer lane)
  bool failed = false;                 // this thread saw a wait time out
  __shared__ int any_failed;           // block-uniform copy, read after barriers
  __shared__ uint32_t s_cnt[kPfQPerBlock];
  if (tid == 0) any_failed = 0;
  for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
    const PfItem x = pf_item(p, it);
    const int64_t n_t = pf_count(p, x);
    // query block -> B operand (all threads), 64-byte swizzle, zero rows past H_I / n_q
    for (int i = tid; i < kPfN * 64; i += kPfThreads) {
      const int r = i >> 6, c = i & 63;
      const int qq = r >> 3, j = r & 7;
      const int t = x.qb * kPfQPerBlock + qq;
      uint8_t v = 0;
      if (j < p.H_I && t < p.n_q) v = p.q[(((int64_t)x.b * p.n_q + t) * p.H_I + j) * kDI + c];
      S.qb[sw64_offset(r, c)] = v;
    }
    for (int i = tid; i < kPfQPerBlock * 8; i += kPfThreads) {
      const int qq = i >> 3, j = i & 7;
      const int t = x.qb * kPfQPerBlock + qq;
      S.wts[i] = (j < p.H_I && t < p.n_q) ? p.w[((int64_t)x.b * p.n_q + t) * p.H_I + j] : 0.f;
    }
    if (tid < kPfQPerBlock) s_cnt[tid] = 0;
    fence_proxy_async_smem();
    __syncthreads();

    if (warp == 0) {
      if (lane == 0 && !failed) {
        for (int64_t i = 0; i < n_t; ++i) {
          const int64_t g = run + i;
          const int s = (int)(g % kPfStages);
          const uint32_t ph = (uint32_t)(g / kPfStages) & 1u;
          if (!mbar_wait(&S.empty[s], ph ^ 1u, &g_pf_error, kErrWaitSmemEmpty)) { failed = true; break; }
          mbar_arrive_expect_tx(&S.full[s], kPfStageBytes);
          tma_load_3d(S.stage + (size_t)s * kPfStageBytes, &tmap, &S.full[s], 0,
                      (int)(pf_tile(p, x, i) * kPfRows), x.b);
          issued = g + 1;
        }
      }
    } else if (warp == 1) {
      if (lane == 0 && !failed) {
        constexpr uint32_t idesc = idesc_make(kFmtE4M3, kFmtE4M3, kPfRows, kPfN);
        const uint64_t bdesc = desc_k_sw64(smem_u32(S.qb));
        for (int64_t i = 0; i < n_t; ++i) {
          const int64_t g = run + i;
          const int s = (int)(g % kPfStages), a = (int)(g % kPfAcc);
          if (!mbar_wait(&S.full[s], (uint32_t)(g / kPfStages) & 1u, &g_pf_error, kErrWaitTmaFull)) { failed = true; break; }
          if (!mbar_wait(&S.acce[a], ((uint32_t)(g / kPfAcc) & 1u) ^ 1u, &g_pf_error, kErrWaitAccEmpty)) { failed = true; break; }
          tc_fence_after();
          const uint64_t adesc = desc_k_sw64(smem_u32(S.stage + (size_t)s * kPfStageBytes));
          const uint32_t d = tbase + (uint32_t)(a * kPfN);
          mma_f8f6f4_ss(d, adesc, bdesc, idesc, 0u);
          mma_f8f6f4_ss(d, adesc + 2, bdesc + 2, idesc, 1u);
          mma_commit(&S.empty[s]);
          mma_commit(&S.accf[a]);
        }
      }
    } else {
      // epilogue warp e: TMEM quarter e % 4 (32 key rows), query group e / 4
      // (8 queries = 64 accumulator columns, all loaded at once: eight
      // independent multiply-add chains, packed two heads per instruction)
      const int e = warp - 2;
      const int quarter = warp & 3;
      const int qg = e >> 2;
      const int t0 = x.qb * kPfQPerBlock + qg * 8;          // first query of the group
      const int64_t row0 = (int64_t)x.b * p.n_q + t0;
      const int lim0 = (int)(p.T - p.n_q) + t0;              // last visible position of query t0
      const int nlive = min(8, p.n_q - t0);
      float tau[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) tau[k] = (MODE == 1 && k < nlive) ? p.tau[row0 + k] : INFINITY;
      // the group's 8 x 8 head weights stay in registers for the whole item,
      // halved: w * relu(x) is computed as (w / 2) * (x + |x|) (see relu2)
      float2 wr[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 v = *reinterpret_cast<const float2*>(S.wts + qg * 64 + 2 * k);
        wr[k] = make_float2(0.5f * v.x, 0.5f * v.y);
      }
      const int kc = (int)(x.kt0 / kPfChunkTiles);
      uint2* cand_base = p.cand + (row0 * p.kchunks + kc) * (int64_t)p.chunk_cap;
      const int nt = (int)n_t;
      const int run32 = (int)(run & 0x7FFFFFFF);
      for (int i = 0; i < nt; ++i) {
        const uint32_t g = (uint32_t)(run32 + i);
        const int a = (int)(g & (kPfAcc - 1));
        if (!mbar_wait(&S.accf[a], (g / kPfAcc) & 1u, &g_pf_error, kErrWaitAccFull)) { failed = true; break; }
        tc_fence_after();
        const uint32_t col0 = tbase + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * kPfN + qg * 64);
        // two halves of 4 queries: one 32-column load each
        float sc[8];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t r32[32];
          tmem_ld32(col0 + 32 * hf, r32);
          tmem_wait_ld();
          if (hf == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acce[a]);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = 4 * hf + kk;
            const uint32_t* rr = r32 + 8 * kk;
            float2 acc = __fmul2_rn(wr[4 * k], relu2(rr[0], rr[1]));
            acc = __ffma2_rn(wr[4 * k + 1], relu2(rr[2], rr[3]), acc);
            acc = __ffma2_rn(wr[4 * k + 2], relu2(rr[4], rr[5]), acc);
            acc = __ffma2_rn(wr[4 * k + 3], relu2(rr[6], rr[7]), acc);
            sc[k] = acc.x + acc.y;
          }
        }
        const int tile = MODE == 1 ? (int)x.kt0 + i : (int)pf_tile(p, x, i);
        const int pos = tile * kPfRows + 32 * quarter + lane;
        // visibility: every position of the tile is visible to every query
        // of the group unless the tile crosses the causal diagonal
        const bool all_vis = tile * kPfRows + kPfRows - 1 <= lim0;
        if (MODE == 0) {
          const int64_t col = (int64_t)(tile / kSampleStride) * kPfRows + 32 * quarter + lane;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k < nlive)
              p.sample[(row0 + k) * p.n_samp + col] = (all_vis || pos <= lim0 + k) ? sc[k] : -INFINITY;
        } else {
          bool any = false;                  // tau = +inf for dead queries: never hits
#pragma unroll
          for (int k = 0; k < 8; ++k) any |= sc[k] >= tau[k];
          if (any) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (sc[k] >= tau[k] && (all_vis || pos <= lim0 + k)) {
                const uint32_t slot = atomicAdd(&s_cnt[qg * 8 + k], 1u);
                if (slot < (uint32_t)p.chunk_cap)
                  cand_base[(int64_t)k * p.kchunks * p.chunk_cap + slot] = make_uint2(order_key(sc[k]), (uint32_t)pos);
              }
            }
          }
        }
      }
    }
    run += n_t;
    if (failed) atomicExch(&any_failed, 1);
    __syncthreads();
    if (MODE == 1 && tid < kPfQPerBlock) {
      const int t = x.qb * kPfQPerBlock + tid;
      if (t < p.n_q) p.cnt[((int64_t)x.b * p.n_q + t) * p.kchunks + x.kt0 / kPfChunkTiles] = s_cnt[tid];
    }
    if (any_failed) break;
  }
  if (warp == 0 && lane == 0) drain_copies(S.full, kPfStages, issued, &g_pf_error, kErrWaitTmaFull);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// tau_t: the smallest of the r best sampled scores, or -inf when every
// visible position fits in the candidate buffer.
__global__ void prefill_tau_kernel(const float* sample, int64_t n_samp, const int32_t* sidx, int r, int rows,
                                   int n_q, int64_t T, int64_t fit, float* tau) {
  pdl_enter();
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const int t = row % n_q;
  const int64_t visible = T - n_q + t + 1;
  float m = INFINITY;
  int have = 0;
  for (int k = 0; k < r; ++k) {
    const int32_t c = sidx[(int64_t)row * r + k];
    if (c >= 0) { m = fminf(m, sample[(int64_t)row * n_samp + c]); ++have; }
  }
  tau[row] = (visible <= fit || have == 0 || m == -INFINITY) ? -INFINITY : m;
}

// ------------------------------------------------------------- final select --
constexpr int kPfFinalThreads = 1024;
constexpr int kPfMaxK = 4096;

template <int NT>
CSA_DEV uint32_t blk_scan(uint32_t v, uint32_t* wt, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) wt[wid] = v;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < NT / 32 ? wt[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < NT / 32) wt[lane] = w;
    if (lane == NT / 32 - 1) *total = w;
  }
  __syncthreads();
  const uint32_t r = v + (wid > 0 ? wt[wid - 1] : 0u);
  __syncthreads();
  return r;
}

// Radix select over (value, mask) pairs held by the block: returns in *out
// the K-th largest value among those with sel(i) true, and in *krem how
// many entries equal to it are needed.  `get(i)` returns the 32-bit value.
template <typename Get, typename Sel>
CSA_DEV void radix_kth(uint32_t n, uint32_t K, Get get, Sel sel, uint32_t* hist, uint32_t* s_prefix,
                       uint32_t* s_krem) {
  const int tid = threadIdx.x;
  if (tid == 0) { *s_prefix = 0; *s_krem = K; }
  __syncthreads();
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kPfFinalThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = *s_prefix;
    for (uint32_t i = tid; i < n; i += kPfFinalThreads) {
      if (!sel(i)) continue;
      const uint32_t k = get(i);
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t loc[8], s = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) { loc[k] = hist[255 - 8 * tid - k]; s += loc[k]; }
      uint32_t inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (tid >= o) inc += t;
      }
      const uint32_t exc = inc - s, krem = *s_krem;
      if (exc < krem && inc >= krem) {
        uint32_t cum = exc;
        for (int k = 0; k < 8; ++k) {
          if (cum + loc[k] >= krem) {
            *s_prefix = prefix | ((255u - 8u * tid - k) << shift);
            *s_krem = krem - cum;
            break;
          }
          cum += loc[k];
        }
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
}

struct PfFinalParams {
  const uint8_t* keys;
  int64_t key_row_stride, key_batch_stride;
  const uint8_t* q;
  const float* w;
  int n_q, H_I, K;
  int64_t T;
  const float* tau;
  const uint2* cand;       // [rows][kchunks][chunk_cap]
  const uint32_t* cnt;     // [rows][kchunks]
  int kchunks;
  int chunk_cap;
  int32_t* idx;            // [B*n_q][K]
};

// Exact score of one key on the CUDA cores (fallback path): E4M3 products are
// exact in fp32 and the 64-term sums are accumulated in fp32, which matches
// the tensor-core result to within fp32 rounding; the fallback selects with
// its own scores, consistently, so its result is the exact Top-K of them.
CSA_DEV float key_score(const uint8_t* krow, const float (*qf)[64], const float (&wv)[8], int H_I) {
  float kf[64];
#pragma unroll
  for (int c = 0; c < 64; c += 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(krow + c);
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 f = __half22float2(dec_e4m3x2((ww[k >> 1] >> (16 * (k & 1))) & 0xFFFF));
      kf[c + 2 * k] = f.x;
      kf[c + 2 * k + 1] = f.y;
    }
  }
  float s = 0.f;
  for (int j = 0; j < H_I; ++j) {
    float d = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) d = fmaf(qf[j][c], kf[c], d);
    s = fmaf(wv[j], fmaxf(d, 0.f), s);
  }
  return s;
}

__global__ void __launch_bounds__(kPfFinalThreads) prefill_final_kernel(PfFinalParams p) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* ck = reinterpret_cast<uint32_t*>(smem);                 // [kCandCap] keys
  uint32_t* cp = ck + kCandCap;                                      // [kCandCap] positions
  uint32_t* bucket = cp + kCandCap;                                  // [kPfMaxK] bucket heads
  uint32_t* outp = bucket + kPfMaxK;                                 // [kPfMaxK] selected positions
  __shared__ uint32_t wt[32], total, hist[256], s_prefix, s_krem, s_prefix2, s_krem2;
  __shared__ float qf_s[8][64];
  const int tid = threadIdx.x;
  const int row = blockIdx.x;
  const int b = row / p.n_q, t = row - b * p.n_q;
  const int64_t visible = p.T - p.n_q + t + 1;
  const uint32_t K = (uint32_t)p.K;
  int32_t* out = p.idx + (int64_t)row * p.K;
  __shared__ uint32_t s_total, s_over;
  if (tid == 0) {
    uint32_t tot = 0, over = 0;
    for (int c = 0; c < p.kchunks; ++c) {
      const uint32_t n = p.cnt[(int64_t)row * p.kchunks + c];
      over |= n > (uint32_t)p.chunk_cap ? 1u : 0u;
      tot += n;
    }
    s_total = tot;
    s_over = over;
  }
  __syncthreads();
  const uint32_t c_all = s_total;
  const float tau = p.tau[row];
  const bool fast = !s_over && c_all <= (uint32_t)kCandCap && (c_all >= K || tau == -INFINITY);

  uint32_t n_sel = 0;    // selected positions gathered into outp (unsorted)
  if (fast) {
    const uint32_t m = c_all;
    {
      uint32_t base = 0;
      for (int c = 0; c < p.kchunks; ++c) {
        const uint32_t n = p.cnt[(int64_t)row * p.kchunks + c];
        const uint2* src = p.cand + ((int64_t)row * p.kchunks + c) * p.chunk_cap;
        for (uint32_t i = tid; i < n; i += kPfFinalThreads) {
          const uint2 v = src[i];
          ck[base + i] = v.x;
          cp[base + i] = v.y;
        }
        base += n;
      }
    }
    __syncthreads();
    const bool take_all = m <= K;
    uint32_t tau_k = 0, need = 0, pos_cut = 0xFFFFFFFFu;
    if (!take_all) {
      radix_kth(m, K, [&](uint32_t i) { return ck[i]; }, [&](uint32_t) { return true; }, hist, &s_prefix, &s_krem);
      tau_k = s_prefix;
      need = s_krem;
      // lowest `need` positions among keys equal to tau_k: the need-th smallest
      // position = the (cnt_eq - need + 1)-th largest of the complemented positions
      radix_kth(m, need, [&](uint32_t i) { return ~cp[i]; }, [&](uint32_t i) { return ck[i] == tau_k; }, hist,
                &s_prefix2, &s_krem2);
      pos_cut = ~s_prefix2;
    }
    // gather the selected positions
    uint32_t mine = 0;
    const uint32_t seg = (m + kPfFinalThreads - 1) / kPfFinalThreads;
    const uint32_t i0 = min(m, tid * seg), i1 = min(m, i0 + seg);
    for (uint32_t i = i0; i < i1; ++i)
      mine += (take_all || ck[i] > tau_k || (ck[i] == tau_k && cp[i] <= pos_cut)) ? 1u : 0u;
    uint32_t o = blk_scan<kPfFinalThreads>(mine, wt, &total) - mine;
    n_sel = total;
    for (uint32_t i = i0; i < i1; ++i)
      if (take_all || ck[i] > tau_k || (ck[i] == tau_k && cp[i] <= pos_cut)) outp[o++] = cp[i];
    __syncthreads();
  } else {
    // exact streaming fallback: 4 radix passes over recomputed scores, then
    // an in-order emission pass (positions come out ascending)
    for (int i = tid; i < 8 * 64; i += kPfFinalThreads) {
      const int j = i >> 6, c = i & 63;
      qf_s[j][c] = j < p.H_I ? dec_e4m3(p.q[(((int64_t)row) * p.H_I + j) * kDI + c]) : 0.f;
    }
    __syncthreads();
    const float (*qf)[64] = qf_s;
    float wv[8];
    for (int j = 0; j < 8; ++j) wv[j] = j < p.H_I ? p.w[(int64_t)row * p.H_I + j] : 0.f;
    const uint8_t* kb = p.keys + (int64_t)b * p.key_batch_stride;
    const uint32_t n = (uint32_t)visible;
    const bool take_all = n <= K;
    uint32_t tau_k = 0, need = K;
    if (!take_all) {
      radix_kth(n, K, [&](uint32_t i) { return order_key(key_score(kb + (int64_t)i * p.key_row_stride, qf, wv, p.H_I)); },
                [&](uint32_t) { return true; }, hist, &s_prefix, &s_krem);
      tau_k = s_prefix;
      need = s_krem;
    }
    uint32_t eq_base = 0, base = 0;
    for (uint32_t i0 = 0; i0 < n; i0 += kPfFinalThreads) {
      const uint32_t i = i0 + tid;
      uint32_t k = 0;
      if (i < n) k = order_key(key_score(kb + (int64_t)i * p.key_row_stride, qf, wv, p.H_I));
      const uint32_t eq = (i < n && !take_all && k == tau_k) ? 1u : 0u;
      const uint32_t eqi = blk_scan<kPfFinalThreads>(eq, wt, &total);
      const uint32_t eqt = total;
      const bool sel = i < n && (take_all || k > tau_k || (eq && eq_base + eqi - 1 < need));
      const uint32_t si = blk_scan<kPfFinalThreads>(sel ? 1u : 0u, wt, &total);
      if (sel) out[base + si - 1] = (int32_t)i;
      base += total;
      eq_base += eqt;
    }
    for (uint32_t j = base + tid; j < K; j += kPfFinalThreads) out[j] = -1;
    return;
  }

  // sort the selected positions ascending: bucket by the top bits, then an
  // insertion sort inside each (small) bucket
  int shift = 0;
  while (((uint64_t)(visible - 1) >> shift) >= (uint64_t)kPfMaxK) ++shift;
  for (int i = tid; i < kPfMaxK; i += kPfFinalThreads) bucket[i] = 0;
  __syncthreads();
  uint32_t* tmp = ck;                         // candidates are no longer needed
  for (uint32_t i = tid; i < n_sel; i += kPfFinalThreads) atomicAdd(&bucket[outp[i] >> shift], 1u);
  __syncthreads();
  {
    // exclusive scan of kPfMaxK bucket counts, 4 per thread
    uint32_t c4[4], s4 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) { c4[k] = bucket[4 * tid + k]; s4 += c4[k]; }
    uint32_t o = blk_scan<kPfFinalThreads>(s4, wt, &total) - s4;
#pragma unroll
    for (int k = 0; k < 4; ++k) { bucket[4 * tid + k] = o; o += c4[k]; }
  }
  __syncthreads();
  // bucket[i] is now the start of bucket i; scatter with a per-bucket cursor in cp
  for (int i = tid; i < kPfMaxK; i += kPfFinalThreads) cp[i] = bucket[i];
  __syncthreads();
  for (uint32_t i = tid; i < n_sel; i += kPfFinalThreads) {
    const uint32_t v = outp[i];
    tmp[atomicAdd(&cp[v >> shift], 1u)] = v;
  }
  __syncthreads();
  for (int bk = tid; bk < kPfMaxK; bk += kPfFinalThreads) {
    const uint32_t lo = bucket[bk], hi = cp[bk];
    for (uint32_t i = lo + 1; i < hi; ++i) {
      const uint32_t v = tmp[i];
      uint32_t j = i;
      while (j > lo && tmp[j - 1] > v) { tmp[j] = tmp[j - 1]; --j; }
      tmp[j] = v;
    }
  }
  __syncthreads();
  for (uint32_t j = tid; j < K; j += kPfFinalThreads) out[j] = j < n_sel ? (int32_t)tmp[j] : -1;
}

// ----------------------------------------------------------------- host --
bool make_key_tmap(CUtensorMap* map, const uint8_t* keys, int64_t T, int B, int64_t row_stride,
                   int64_t batch_stride);

struct PfWs {
  float* sample;
  SelectJob sel;
  int32_t* sidx;
  float* tau;
  uint2* cand;
  uint32_t* cnt;
  size_t bytes;
};

static size_t al256p(size_t x) { return (x + 255) & ~(size_t)255; }

static int pf_sample_r(int K) {
  // keep ~2K positions: r = 2K / kSampleStride sampled ranks (at least 4)
  int r = (2 * K + kSampleStride - 1) / kSampleStride;
  return r < 4 ? 4 : r;
}

// Candidates kept per (query, key chunk): ~2K are expected per query in
// total, spread over the chunks; keep a wide margin, at least 2048.
static int pf_chunk_cap(int64_t ntiles) {
  const int kchunks = (int)((ntiles + kPfChunkTiles - 1) / kPfChunkTiles);
  int cap = 16384 / (kchunks > 0 ? kchunks : 1);
  if (cap < 2048) cap = 2048;
  if (cap > kChunkCapMax) cap = kChunkCapMax;
  return cap;
}

static PfWs carve_pf_ws(const csa_index_args* a, void* ws) {
  PfWs w{};
  const int rows = a->B * a->n_q;
  const int64_t ntiles = (a->T + kPfRows - 1) / kPfRows;
  const int64_t n_samp = ((ntiles + kSampleStride - 1) / kSampleStride) * kPfRows;
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = 0;
  auto take = [&](size_t n) { uint8_t* p = base ? base + off : nullptr; off += al256p(n); return p; };
  w.sample = reinterpret_cast<float*>(take((size_t)rows * n_samp * 4));
  off += select_carve(w.sel, rows, n_samp, base ? base + off : nullptr);
  w.sidx = reinterpret_cast<int32_t*>(take((size_t)rows * pf_sample_r(a->K) * 4));
  w.tau = reinterpret_cast<float*>(take((size_t)rows * 4));
  const int kchunks = (int)((ntiles + kPfChunkTiles - 1) / kPfChunkTiles);
  w.cnt = reinterpret_cast<uint32_t*>(take((size_t)rows * kchunks * 4));
  w.cand = reinterpret_cast<uint2*>(take((size_t)rows * kchunks * pf_chunk_cap(ntiles) * 8));
  w.bytes = off;
  return w;
}

size_t index_prefill_ws_bytes(const csa_index_args* a) { return carve_pf_ws(a, nullptr).bytes; }

cudaError_t run_index_prefill(const csa_index_args* a, void* ws, cudaStream_t stream) {
  PfWs w = carve_pf_ws(a, ws);
  const int rows = a->B * a->n_q;
  const int64_t ntiles = (a->T + kPfRows - 1) / kPfRows;
  const int64_t n_samp = ((ntiles + kSampleStride - 1) / kSampleStride) * kPfRows;
  const int r = pf_sample_r(a->K);
  cudaError_t e;
  CUtensorMap map;
  if (!make_key_tmap(&map, a->keys, a->T, a->B, a->key_row_stride, a->key_batch_stride))
    return cudaErrorInvalidValue;
  e = launch_zero(w.sel.hist, (size_t)rows * kHistBins * 4, stream);
  if (e != cudaSuccess) return e;

  static SmemAttrOnce attr0, attr1, attr_final;
  if ((e = attr0.set(prefill_score_tc_kernel<0>, kPfSmemBytes)) != cudaSuccess) return e;
  if ((e = attr1.set(prefill_score_tc_kernel<1>, kPfSmemBytes)) != cudaSuccess) return e;
  if ((e = attr_final.set(prefill_final_kernel, (size_t)(2 * kCandCap + 2 * kPfMaxK) * 4)) != cudaSuccess) return e;
  PfParams p{};
  p.q = a->q;
  p.w = a->w;
  p.B = a->B;
  p.n_q = a->n_q;
  p.H_I = a->H_I;
  p.T = a->T;
  p.qblocks = (a->n_q + kPfQPerBlock - 1) / kPfQPerBlock;
  p.ntiles = ntiles;
  p.kchunks = (int)((ntiles + kPfChunkTiles - 1) / kPfChunkTiles);
  p.n_items = a->B * p.qblocks * p.kchunks;
  p.sample = w.sample;
  p.n_samp = n_samp;
  p.tau = w.tau;
  p.cand = w.cand;
  p.cnt = w.cnt;
  p.chunk_cap = pf_chunk_cap(ntiles);
  const int grid = p.n_items < kNumSMs ? p.n_items : kNumSMs;

  // 1. sample pass + per-query threshold
  p.mode = 0;
  {
    ProfScope ps(stream, "prefill_score_tc[sample]");
    launch_k(prefill_score_tc_kernel<0>, dim3(grid), dim3(kPfThreads), kPfSmemBytes, stream, map, p);
  }
  note_launches(1);
  SelectJob& j = w.sel;
  j.vals = w.sample;
  j.row_stride = n_samp;
  j.n_row = nullptr;
  j.K = r;
  j.out = w.sidx;
  j.out_stride = r;
  j.out_width = r;
  j.map = nullptr;
  j.expand = 0;
  j.out_len = nullptr;
  e = launch_select(&j, 1, rows, true, stream);
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(stream, "prefill_tau");
    // a query whose visible positions all fit in one key chunk's buffer takes
    // every position (tau = -inf); with several chunks, each chunk holds its share
    const int64_t fit = p.kchunks == 1 ? (int64_t)p.chunk_cap : 0;
    launch_k(prefill_tau_kernel, dim3((rows + 255) / 256), dim3(256), 0, stream, w.sample, n_samp, w.sidx, r, rows, a->n_q, a->T, fit,
                                                               w.tau);
  }
  note_launches(1);
  // 2. main pass
  p.mode = 1;
  {
    ProfScope ps(stream, "prefill_score_tc[main]");
    launch_k(prefill_score_tc_kernel<1>, dim3(grid), dim3(kPfThreads), kPfSmemBytes, stream, map, p);
  }
  note_launches(1);
  // 3. exact per-query Top-K
  PfFinalParams f{};
  f.keys = a->keys;
  f.key_row_stride = a->key_row_stride;
  f.key_batch_stride = a->key_batch_stride;
  f.q = a->q;
  f.w = a->w;
  f.n_q = a->n_q;
  f.H_I = a->H_I;
  f.K = a->K;
  f.T = a->T;
  f.tau = w.tau;
  f.cand = w.cand;
  f.cnt = w.cnt;
  f.kchunks = p.kchunks;
  f.chunk_cap = p.chunk_cap;
  f.idx = a->idx;
  {
    ProfScope ps(stream, "prefill_final");
    launch_k(prefill_final_kernel, dim3(rows), dim3(kPfFinalThreads), (2 * kCandCap + 2 * kPfMaxK) * 4, stream, f);
  }
  note_launches(1);
  return cudaGetLastError();
}

int read_pf_error(bool clear) {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_pf_error, sizeof(int));
  if (clear && v) {
    int z = 0;
    cudaMemcpyToSymbol(g_pf_error, &z, sizeof(int));
  }
  return v;
}

}  // namespace csa
