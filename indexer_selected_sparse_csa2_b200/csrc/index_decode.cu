// Lightning-indexer scoring for decode (one query token per sequence).
//
// S[s] = sum_j w[j] * relu(<qI[j], kI[s]>) over FP8 E4M3 keys (Model
// techniques map - DeepSeek-V4.1-Flash, "Indexer-selected sparse attention"
// row: an indexer with its own heads scores the cached tokens; the
// DeepSeek-V4.1-Flash architecture database keeps one indexer key per
// position).  Decode scoring reads 64 B per position and does 16 flop per
// byte (8 heads), which is more than the fp32 CUDA cores sustain at HBM
// speed, so the dot products run on the FP8 tensor-core path:
// mma.sync m16n8k32 e4m3 x e4m3 -> fp32, keys as the M=16 rows, heads as
// N=8.  A thread loads 16 contiguous key bytes of two rows (rows g and g+8 of
// the tile, bytes [16t, 16t+16)); the reduction order over the 64 key bytes
// is permuted identically for the query fragment, which leaves the dot
// product unchanged.
//
// Fused epilogue: ReLU, head weights, head sum (quad shuffles), fp32 score
// store, a 4096-bin shared-memory histogram of the score's order key (first
// radix level of the Top-K select) and, when building the hierarchical pool,
// the max over aligned blocks of positions and that value's histogram.
#include "select.cuh"

namespace csa {

struct ScoreParams {
  const uint8_t* keys;
  int64_t key_row_stride;
  int64_t key_batch_stride;
  const uint8_t* q;          // [B][H_I][64] (n_q == 1)
  const float* w;            // [B][H_I]
  int H_I;
  const int32_t* pool;       // optional [B][pool_cap] slot -> position
  const int32_t* pool_len;   // [B]
  int64_t n;                 // slots per row (T, or pool_cap)
  int64_t chunk;             // slots per CTA (multiple of 512)
  float* scores;             // [B][n]
  uint32_t* hist;            // [B][4096]
  float* bmax;               // optional [B][nb]
  uint32_t* bhist;           // [B][4096]
  int64_t nb;
  int block_len;             // 1, 2, 4, 8 or 16
};

CSA_DEV void mma_e4m3_16832(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kScoreThreads = 256;
constexpr int kTilesPerIter = 4;                       // 4 x 16 rows per warp step
constexpr int kRowsPerIter = 16 * kTilesPerIter;       // 64
constexpr int kRowsPerCtaIter = kRowsPerIter * (kScoreThreads / 32);   // 512

__global__ void __launch_bounds__(kScoreThreads, 2) index_score_decode_kernel(ScoreParams p) {
  pdl_enter();
  __shared__ uint32_t h[kHistBins];
  __shared__ uint32_t hb[kHistBins];
  const int b = blockIdx.y;
  const bool build = p.bmax != nullptr;
  for (int i = threadIdx.x; i < kHistBins; i += kScoreThreads) { h[i] = 0; if (build) hb[i] = 0; }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  // query fragment: head g, key bytes [16t, 16t+16)
  uint32_t qf[4] = {0u, 0u, 0u, 0u};
  if (g < p.H_I) {
    uint4 v = ld_v4(p.q + ((int64_t)b * p.H_I + g) * kDI + 16 * t);
    qf[0] = v.x; qf[1] = v.y; qf[2] = v.z; qf[3] = v.w;
  }
  const float w0 = (2 * t < p.H_I) ? p.w[(int64_t)b * p.H_I + 2 * t] : 0.f;
  const float w1 = (2 * t + 1 < p.H_I) ? p.w[(int64_t)b * p.H_I + 2 * t + 1] : 0.f;

  const int64_t n_valid = p.pool ? (int64_t)min((int64_t)p.pool_len[b], p.n) : p.n;
  const int64_t lo = (int64_t)blockIdx.x * p.chunk;
  const int64_t hi = min(lo + p.chunk, n_valid);
  const uint8_t* kb = p.keys + (int64_t)b * p.key_batch_stride;
  const int32_t* pl = p.pool ? p.pool + (int64_t)b * p.n : nullptr;
  float* sc = p.scores + (int64_t)b * p.n;
  __syncthreads();

  // Register double buffer: the loads of the warp's next 64 rows are issued
  // before the current 64 rows are multiplied, so every warp keeps 4 KB of
  // key reads in flight while it computes.
  uint4 ka[2][kTilesPerIter], kc[2][kTilesPerIter];
  auto load = [&](int buf, int64_t base) {
#pragma unroll
    for (int u = 0; u < kTilesPerIter; ++u) {
      const int64_t r0 = base + 16 * u + g, r1 = r0 + 8;
      ka[buf][u] = make_uint4(0, 0, 0, 0);
      kc[buf][u] = make_uint4(0, 0, 0, 0);
      if (r0 < hi) {
        const int64_t s0 = pl ? (int64_t)pl[r0] : r0;
        ka[buf][u] = ld_nc_v4(kb + s0 * p.key_row_stride + 16 * t);
      }
      if (r1 < hi) {
        const int64_t s1 = pl ? (int64_t)pl[r1] : r1;
        kc[buf][u] = ld_nc_v4(kb + s1 * p.key_row_stride + 16 * t);
      }
    }
  };
  auto compute = [&](int buf, int64_t base) {
#pragma unroll
    for (int u = 0; u < kTilesPerIter; ++u) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const uint4 A = ka[buf][u], C = kc[buf][u];
      mma_e4m3_16832(c, A.x, C.x, A.y, C.y, qf[0], qf[1]);
      mma_e4m3_16832(c, A.z, C.z, A.w, C.w, qf[2], qf[3]);
      float s_lo = w0 * fmaxf(c[0], 0.f) + w1 * fmaxf(c[1], 0.f);   // row g
      float s_hi = w0 * fmaxf(c[2], 0.f) + w1 * fmaxf(c[3], 0.f);   // row g + 8
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
      const int64_t tile = base + 16 * u;
      const int64_t r_lo = tile + g, r_hi = r_lo + 8;
      if (t == 0 && r_lo < hi) {
        sc[r_lo] = s_lo;
        atomicAdd(&h[order_key(s_lo) >> (32 - kHistBits)], 1u);
      }
      if (t == 1 && r_hi < hi) {
        sc[r_hi] = s_hi;
        atomicAdd(&h[order_key(s_hi) >> (32 - kHistBits)], 1u);
      }
      if (build) {
        // block max over aligned groups of block_len rows (rows g and g+8 of the tile)
        float m_lo = r_lo < hi ? s_lo : -INFINITY;
        float m_hi = r_hi < hi ? s_hi : -INFINITY;
        const int bl = p.block_len;
        if (bl >= 2) { m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 4)); m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 4)); }
        if (bl >= 4) { m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 8)); m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 8)); }
        if (bl >= 8) { m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 16)); m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 16)); }
        if (bl >= 16) m_lo = m_hi = fmaxf(m_lo, m_hi);
        // the quad holding a block's first row publishes it (lane 0: row
        // g, lane 1: row g + 8); chunks are multiples of 16 rows, so a block
        // never straddles two CTAs
        if (bl < 16) {
          if ((g % bl) == 0 && t < 2) {
            const int64_t row = tile + g + 8 * t;
            const float m = t ? m_hi : m_lo;
            if (row < hi) {
              p.bmax[(int64_t)b * p.nb + row / bl] = m;
              atomicAdd(&hb[order_key(m) >> (32 - kHistBits)], 1u);
            }
          }
        } else if (lane == 0 && tile < hi) {
          p.bmax[(int64_t)b * p.nb + tile / 16] = m_lo;
          atomicAdd(&hb[order_key(m_lo) >> (32 - kHistBits)], 1u);
        }
      }
    }
  };
  // two iterations per loop trip so that the buffer index is a constant
  int64_t base = lo + (int64_t)warp * kRowsPerIter;
  if (base < hi) load(0, base);
  while (base < hi) {
    int64_t next = base + kRowsPerCtaIter;
    if (next < hi) load(1, next);
    compute(0, base);
    base = next;
    if (base >= hi) break;
    next = base + kRowsPerCtaIter;
    if (next < hi) load(0, next);
    compute(1, base);
    base = next;
  }
  __syncthreads();
  uint32_t* gh = p.hist + (int64_t)b * kHistBins;
  uint32_t* gbh = build ? p.bhist + (int64_t)b * kHistBins : nullptr;
  for (int i = threadIdx.x; i < kHistBins; i += kScoreThreads) {
    if (h[i]) atomicAdd(&gh[i], h[i]);
    if (build && hb[i]) atomicAdd(&gbh[i], hb[i]);
  }
}

int64_t score_chunk(int B, int64_t n) {
  // one wave: two resident CTAs per SM over all rows
  int64_t target = ((int64_t)kNumSMs * 2 + B - 1) / (B > 0 ? B : 1);
  if (target < 1) target = 1;
  int64_t c = (n + target - 1) / target;
  c = (c + kRowsPerCtaIter - 1) / kRowsPerCtaIter * kRowsPerCtaIter;
  if (c < kRowsPerCtaIter) c = kRowsPerCtaIter;
  return c;
}

cudaError_t launch_score_decode(const ScoreParams& p, int B, cudaStream_t stream) {
  const int nchunks = (int)((p.n + p.chunk - 1) / p.chunk);
  dim3 grid(nchunks > 0 ? nchunks : 1, B);
  ProfScope ps(stream, p.pool ? "index_score_decode[pool]" : "index_score_decode[full]");
  launch_k(index_score_decode_kernel, dim3(grid), dim3(kScoreThreads), 0, stream, p);
  note_launches(1);
  return cudaGetLastError();
}

// ----------------------------------------------------------- entry point --
struct IndexWs {
  uint32_t* hist;            // [B][4096] first-level histogram of the scores
  uint32_t* bhist;           // [B][4096] ... of the block maxima (pool build)
  float* scores;             // [B][n] (unless the caller takes them)
  float* bmax;               // [B][nb] block maxima (pool build)
  size_t bytes;
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

cudaError_t launch_score_tc(const csa_index_args* a, float* scores, uint32_t* hist, float* bmax, uint32_t* bhist,
                            int64_t nb, int64_t safe_rows, cudaStream_t stream);
cudaError_t launch_score_mx(const csa_index_args* a, float* scores, uint32_t* hist, float* bmax, uint32_t* bhist,
                            int64_t nb, bool q_early, cudaStream_t stream);

// Pool searches whose slots fit the fused cluster kernel score and select in
// one launch and need no workspace.
static bool fused_pool(const csa_index_args* a) { return a->pool && cs_pool_ok(a->pool_cap); }

// Workspace layout of one decode index call.
static IndexWs carve_index_ws(const csa_index_args* a, void* ws) {
  IndexWs w{};
  const int B = a->B;
  const int64_t n = a->pool ? (int64_t)a->pool_cap : a->T;
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = 0;
  // both first-level histograms side by side, cleared by one launch
  w.hist = reinterpret_cast<uint32_t*>(base);
  w.bhist = w.hist + (size_t)B * kHistBins;
  off += al256((size_t)2 * B * kHistBins * 4);
  if (!fused_pool(a)) {
    w.scores = reinterpret_cast<float*>(base + off);
    off += al256((size_t)B * n * 4);
  }
  if (a->pool_out) {
    const int64_t nb = (a->T + a->pool_block_len - 1) / a->pool_block_len;
    w.bmax = reinterpret_cast<float*>(base + off);
    off += al256((size_t)B * nb * 4);
  }
  w.bytes = off;
  return w;
}

size_t index_prefill_ws_bytes(const csa_index_args* a);
cudaError_t run_index_prefill(const csa_index_args* a, void* ws, cudaStream_t stream);

size_t index_decode_ws_bytes(const csa_index_args* a) {
  if (a->n_q > 1) return index_prefill_ws_bytes(a);
  return carve_index_ws(a, nullptr).bytes;
}

size_t index_hist_bytes(const csa_index_args* a) {
  return a->n_q > 1 ? 0 : al256((size_t)2 * a->B * kHistBins * 4);
}

// `hists`: optional region of index_hist_bytes(a) that the caller has already
// cleared (a layer stack clears all its layers' histograms in one launch);
// without it the workspace's own histograms are cleared here.  `pool_done`:
// optional event recorded once the candidate pool is written (before the
// position Top-K of a pool-building call), so that layers searching the pool
// can start early.  `safe_rows` (used with `hists` only, i.e. inside a layer
// stack right after its prologue kernel): key rows below it, and the query and
// head weights, are not written by that prologue, so the full scan may read
// them before waiting for it; < 0 waits first.
cudaError_t run_index_decode(const csa_index_args* a, void* ws, cudaStream_t stream, uint32_t* hists,
                             cudaEvent_t pool_done, int64_t safe_rows) {
  if (a->n_q > 1) return run_index_prefill(a, ws, stream);
  IndexWs w = carve_index_ws(a, ws);
  const int B = a->B;
  const int64_t n = a->pool ? (int64_t)a->pool_cap : a->T;
  cudaError_t e;
  float* scores = a->scores ? a->scores : w.scores;

  CsRow jp{};
  jp.n = n;
  jp.K = a->K;
  jp.out = a->idx;
  jp.out_stride = a->K;
  jp.out_width = a->K;
  jp.run = cs_run(n);
  if (fused_pool(a)) {
    // Reindex inside the pool: gather + score + select in one cluster launch
    jp.row_stride = a->pool_cap;
    jp.map = a->pool;
    jp.map_stride = a->pool_cap;
    CsPool pp{};
    pp.keys = a->keys;
    pp.key_row_stride = a->key_row_stride;
    pp.key_batch_stride = a->key_batch_stride;
    pp.q = a->q;
    pp.w = a->w;
    pp.H_I = a->H_I;
    pp.pool_len = a->pool_len;
    pp.scores = a->scores;
    return launch_cluster_pool_select(jp, pp, B, stream);
  }

  if (hists) {
    w.hist = hists;
    w.bhist = hists + (size_t)B * kHistBins;
  } else {
    // histograms start at zero (both sit at the start of the workspace)
    e = launch_zero(w.hist, (size_t)(a->pool_out ? 2 : 1) * B * kHistBins * 4, stream);
    if (e != cudaSuccess) return e;
  }
  const int64_t nb = a->pool_out ? (a->T + a->pool_block_len - 1) / a->pool_block_len : 0;
  // a pool-building call whose Top-K is taken inside the pool never reads the
  // positions' histogram: the scorer skips it
  const int64_t pool_cap = (int64_t)a->pool_blocks * a->pool_block_len;
  const bool topk_in_pool = a->pool_out && a->pool_blocks >= a->K && cs_pool_ok(pool_cap);
  uint32_t* pos_hist = topk_in_pool ? nullptr : w.hist;
  if (a->pool) {
    // pool rows too long for the fused kernel: gathered scoring, then the select
    ScoreParams p{};
    p.keys = a->keys;
    p.key_row_stride = a->key_row_stride;
    p.key_batch_stride = a->key_batch_stride;
    p.q = a->q;
    p.w = a->w;
    p.H_I = a->H_I;
    p.pool = a->pool;
    p.pool_len = a->pool_len;
    p.n = n;
    p.chunk = score_chunk(B, n);
    p.scores = scores;
    p.hist = w.hist;
    e = launch_score_decode(p, B, stream);
  } else if (a->key_format == CSA_KEY_MXFP4) {
    e = launch_score_mx(a, scores, pos_hist, w.bmax, w.bhist, nb, hists && safe_rows >= 0, stream);
  } else {
    e = launch_score_tc(a, scores, pos_hist, w.bmax, w.bhist, nb, hists ? safe_rows : -1, stream);
  }
  if (e != cudaSuccess) return e;

  if (a->pool_out) {
    // the candidate pool first: the pool layers wait only for it
    CsRow jb{};
    jb.vals = w.bmax;
    jb.row_stride = nb;
    jb.vec = (nb % 4) == 0;
    jb.n = nb;
    jb.hist = w.bhist;
    jb.K = a->pool_blocks;
    jb.out = a->pool_out;
    jb.out_stride = (int64_t)a->pool_blocks * a->pool_block_len;
    jb.out_width = a->pool_blocks * a->pool_block_len;
    jb.expand = a->pool_block_len;
    jb.out_len = a->pool_out_len;
    jb.limit = a->T;
    jb.run = cs_run(nb);
    e = launch_cluster_select(&jb, 1, B, stream, "pool_select");
    if (e != cudaSuccess) return e;
    if (pool_done && cudaEventRecord(pool_done, stream) != cudaSuccess) return cudaErrorUnknown;
  }
  if (topk_in_pool) {
    // The K best positions lie in the pool once it keeps >= K blocks: take any
    // of them, p, in block c.  Were c outside the pool, the pool's blocks
    // would all rank above c (larger max, or the same max and a lower block),
    // and each block's first position holding its max would rank above p
    // (larger score, or the same score at a lower position): pool_blocks >= K
    // positions ahead of p, so p would not be among the K best.  Selecting
    // over the pool's positions (scores gathered by position) is therefore
    // the same as selecting over all T, ties included.
    jp.row_stride = pool_cap;
    jp.n = pool_cap;
    jp.map = a->pool_out;
    jp.map_stride = pool_cap;
    CsPool pp{};
    pp.pool_len = a->pool_out_len;
    pp.gscores = scores;
    pp.gscore_stride = a->T;
    return launch_cluster_pool_select(jp, pp, B, stream);
  }
  jp.vals = scores;
  jp.row_stride = n;
  jp.vec = (n % 4) == 0 && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  jp.n_row = a->pool ? a->pool_len : nullptr;
  jp.hist = w.hist;
  jp.map = a->pool;
  jp.map_stride = a->pool_cap;
  return launch_cluster_select(&jp, 1, B, stream, "topk_select");
}

}  // namespace csa
