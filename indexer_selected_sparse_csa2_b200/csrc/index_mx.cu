// Lightning-indexer scores over MXFP4 indexer keys on the tcgen05 tensor
// cores: the pages' production indexer (Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row: 32 heads of
// dimension 128; DeepSeek-V4.1-Flash architecture database, indexer K
// storage: E2M1 elements with one E8M0 scale per 32 channels, 68 bytes per
// entry), with plain E4M3 queries.
//   S[s] = sum_j w[j] * relu( sum_b 2^(e[s,b]) * <q[j, block b], k[s, block b]> )
// where k is the key's E2M1 codes and e its block exponents.
// Keys sit in two planes: codes [B][T][64 B] and exponent bytes [B][T][4].
//   warp 0     TMA producer: 128-key tiles of the code plane, copied with the
//              packed 4-bit tensor-map type that gives every 16 codes (8
//              bytes) a 16-byte slot in shared memory: the layout in which
//              tcgen05.mma kind::f8f6f4 reads E2M1 operands (one byte of
//              address space per element), 128-byte swizzled; 4 stages;
//   warp 1     MMA issuer: per tile, one tcgen05.mma kind::f8f6f4 per 32-channel
//              block (A = E2M1 keys, M = 128; B = E4M3 queries, N = 32 heads;
//              K = 32) into its own TMEM accumulator (4 x 32 columns per
//              tile, two tiles in flight);
//   warps 2-5  epilogue: one key per thread, the 4 x 32 block dots from
//              TMEM, times 2^e per block, ReLU, head weights, the fp32 score,
//              the first-level Top-K histogram and, when building the pool,
//              the block maxima.
// No thread converts a code: the copy engine spreads them and the tensor
// cores read E2M1 as it is stored.  Two CTAs share each SM (about 100 KB of
// shared memory and 256 TMEM columns each): one CTA's copies land one tile
// per ~0.43 us, so a second CTA doubles the loads in flight per SM.
// All waits are bounded (sm100.cuh).
#include "sm100.cuh"
#include "select.cuh"

namespace csa {

constexpr int kMxRows = 128;                    // keys per tile
constexpr int kMxHeads = 32;
constexpr int kMxStages = 4;
constexpr int kMxStageBytes = kMxRows * 128;    // 16 KB of shared memory per tile (16-byte slot per 16 codes)
constexpr uint32_t kMxStageTx = kMxRows * 64;   // bytes the copy counts: the packed codes
constexpr int kMxEpiGroups = 1;
constexpr int kMxAcc = 2;
constexpr uint32_t kMxTmemCols = 128 * kMxAcc;  // kMxAcc x 4 blocks x 32 heads
constexpr int kMxEpiWarp0 = 2;
constexpr int kMxThreads = 32 * kMxEpiWarp0 + 128 * kMxEpiGroups;
constexpr size_t kMxSmemBytes = 1024 + (size_t)kMxStages * kMxStageBytes + kMxHeads * 128 + 2 * kHistBins * 4 +
                                2 * (kMxStages + kMxAcc) * 8 + 16;
static_assert(2 * (kMxSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");

static __device__ int g_mx_error;

struct MxScoreParams {
  const uint8_t* q;         // [B][32][128] E4M3
  const float* w;           // [B][32]
  const uint8_t* scales;    // exponent bytes, key s of sequence b at scales + b*sbs + s*srs (4 bytes)
  int64_t scale_row_stride, scale_batch_stride;
  int64_t T;
  int tiles_per_cta;
  float* scores;            // [B][T]
  uint32_t* hist;           // [B][4096]
  float* bmax;              // optional [B][nb]
  uint32_t* bhist;
  int64_t nb;
  int block_len;
  int q_early;              // q and w may be read before the wait on the previous kernel
};

__global__ void __launch_bounds__(kMxThreads, 2)
index_score_mx_kernel(const __grid_constant__ CUtensorMap tmap, MxScoreParams p) {
  // the set-up (barriers, histogram clearing, TMEM, and the queries when no
  // appended row of the step writes them) overlaps the previous kernel; keys,
  // exponents and the global histograms are touched only after the wait
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* stage = base;
  uint8_t* qb = stage + (size_t)kMxStages * kMxStageBytes;
  uint32_t* h = reinterpret_cast<uint32_t*>(qb + kMxHeads * 128);
  uint32_t* hb = h + kHistBins;
  uint64_t* bars = reinterpret_cast<uint64_t*>(hb + kHistBins);
  uint64_t* full = bars;                       // [kMxStages] TMA -> MMA
  uint64_t* empty = full + kMxStages;          // [kMxStages] MMA -> TMA
  uint64_t* accf = empty + kMxStages;          // [kMxAcc] MMA -> epilogue
  uint64_t* acce = accf + kMxAcc;              // [kMxAcc] epilogue -> MMA (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + kMxAcc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y;
  const int64_t ntiles_row = (p.T + kMxRows - 1) / kMxRows;
  const int64_t tile0 = (int64_t)blockIdx.x * p.tiles_per_cta;
  const int64_t tile1 = min(tile0 + p.tiles_per_cta, ntiles_row);
  const int n_my = tile1 > tile0 ? (int)(tile1 - tile0) : 0;
  const bool build = p.bmax != nullptr;

  if (tid == 0) {
    for (int i = 0; i < kMxStages; ++i) { mbar_init(full + i, 1); mbar_init(empty + i, 1); }
    for (int i = 0; i < kMxAcc; ++i) { mbar_init(accf + i, 1); mbar_init(acce + i, 4); }
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  for (int i = tid; i < kHistBins; i += kMxThreads) { h[i] = 0; hb[i] = 0; }
  // queries: the B operand, 32 rows of 128 bytes, 128-byte swizzle
  auto stage_q = [&]() {
    for (int i = tid; i < kMxHeads * 8; i += kMxThreads) {
      const int r = i >> 3, c = i & 7;
      const uint4 v = ld_v4(p.q + ((int64_t)b * kMxHeads + r) * 128 + 16 * c);
      *reinterpret_cast<uint4*>(qb + r * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
  };
  if (p.q_early) stage_q();
  if (warp == 1) tmem_alloc(tmem_slot, kMxTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  if (!p.q_early) {
    stage_q();
    __syncthreads();
  }
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kMxStages;
        if (!mbar_wait(empty + s, ((uint32_t)(i / kMxStages) & 1u) ^ 1u, &g_mx_error, kErrWaitSmemEmpty)) break;
        mbar_arrive_expect_tx(full + s, kMxStageTx);
        tma_load_3d(stage + (size_t)s * kMxStageBytes, &tmap, full + s, 0, (int)((tile0 + i) * kMxRows), b);
        issued = i + 1;
      }
      drain_copies(full, kMxStages, issued, &g_mx_error, kErrWaitTmaFull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_make(kFmtE2M1, kFmtE4M3, kMxRows, kMxHeads);
      const uint32_t qa = smem_u32(qb);
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kMxStages, a = i % kMxAcc;
        if (!mbar_wait(full + s, (uint32_t)(i / kMxStages) & 1u, &g_mx_error, kErrWaitTmaFull)) break;
        if (!mbar_wait(acce + a, ((uint32_t)(i / kMxAcc) & 1u) ^ 1u, &g_mx_error, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(stage + (size_t)s * kMxStageBytes);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk)
          mma_f8f6f4_ss(tbase + (uint32_t)(a * 128 + 32 * blk), desc_k_sw128(sa + 32u * blk),
                        desc_k_sw128(qa + 32u * blk), idesc, 0u);
        mma_commit(empty + s);
        mma_commit(accf + a);
      }
    }
  } else {
    // ---- epilogue: group g takes tiles g, g + G, ...; warp w reads TMEM
    // lanes 32 * (w % 4) .. + 31 = keys of the tile
    const int quarter = warp & 3;
    const int grp = (warp - kMxEpiWarp0) >> 2;
    float wj[kMxHeads];
#pragma unroll
    for (int j = 0; j < kMxHeads; ++j) wj[j] = p.w[(int64_t)b * kMxHeads + j];
    float* sc = p.scores + (int64_t)b * p.T;
    const uint8_t* scb = p.scales + (int64_t)b * p.scale_batch_stride;
    const int bl = p.block_len;
    // exponent bytes of this lane's key, loaded one tile of this group ahead
    // (a load at the top of each tile would expose its latency every tile)
    auto exps = [&](int i) -> uint32_t {
      const int64_t r = (tile0 + i) * kMxRows + 32 * quarter + lane;
      return (i < n_my && r < p.T) ? *reinterpret_cast<const uint32_t*>(scb + r * p.scale_row_stride) : 0x7F7F7F7Fu;
    };
    uint32_t e_next = exps(grp);
    for (int i = grp; i < n_my; i += kMxEpiGroups) {
      const int a = i % kMxAcc;
      const int64_t row = (tile0 + i) * kMxRows + 32 * quarter + lane;
      const bool valid = row < p.T;
      const uint32_t ebytes = e_next;
      e_next = exps(i + kMxEpiGroups);
      if (!__all_sync(0xffffffffu, mbar_wait(accf + a, (uint32_t)(i / kMxAcc) & 1u, &g_mx_error, kErrWaitAccFull))) break;
      tc_fence_after();
      float dot[kMxHeads];
#pragma unroll
      for (int j = 0; j < kMxHeads; ++j) dot[j] = 0.f;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
        tmem_ld32(tbase + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * 128 + 32 * blk), v);
        tmem_wait_ld();
        const int e = (int)((ebytes >> (8 * blk)) & 0xFF) - 127;
        const float s2 = e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << 22);
#pragma unroll
        for (int j = 0; j < kMxHeads; ++j) dot[j] = fmaf(__uint_as_float(v[j]), s2, dot[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce + a);
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < kMxHeads; ++j) s = fmaf(wj[j], fmaxf(dot[j], 0.f), s);
      if (valid) {
        sc[row] = s;
        if (p.hist) atomicAdd(&h[order_key(s) >> (32 - kHistBits)], 1u);
      }
      if (build) {
        float m = valid ? s : -INFINITY;
        for (int o = 1; o < bl; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((lane % bl) == 0 && valid) {
          p.bmax[(int64_t)b * p.nb + row / bl] = m;
          atomicAdd(&hb[order_key(m) >> (32 - kHistBits)], 1u);
        }
      }
    }
  }
  __syncthreads();
  uint32_t* gh = p.hist ? p.hist + (int64_t)b * kHistBins : nullptr;
  uint32_t* gbh = build ? p.bhist + (int64_t)b * kHistBins : nullptr;
  for (int i = tid; i < kHistBins; i += kMxThreads) {
    if (gh && h[i]) atomicAdd(&gh[i], h[i]);
    if (build && hb[i]) atomicAdd(&gbh[i], hb[i]);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kMxTmemCols);
  }
}

bool make_key_tmap_e2m1(CUtensorMap* map, const uint8_t* keys, int64_t T, int B, int64_t row_stride,
                        int64_t batch_stride, int box_rows);

cudaError_t launch_score_mx(const csa_index_args* a, float* scores, uint32_t* hist, float* bmax, uint32_t* bhist,
                            int64_t nb, bool q_early, cudaStream_t stream) {
  CUtensorMap map;
  if (!make_key_tmap_e2m1(&map, a->keys, a->T, a->B, a->key_row_stride, a->key_batch_stride, kMxRows))
    return cudaErrorInvalidValue;
  MxScoreParams p{};
  p.q = a->q;
  p.w = a->w;
  p.scales = a->key_scales;
  p.scale_row_stride = a->key_scale_row_stride;
  p.scale_batch_stride = a->key_scale_batch_stride;
  p.T = a->T;
  const int64_t ntiles = (a->T + kMxRows - 1) / kMxRows;
  // one wave of two CTAs per SM (rounded down, so that no CTA waits for a
  // second wave)
  int64_t ctas_row = 2 * kNumSMs / a->B;
  if (ctas_row > ntiles) ctas_row = ntiles;
  if (ctas_row < 1) ctas_row = 1;
  p.tiles_per_cta = (int)((ntiles + ctas_row - 1) / ctas_row);
  ctas_row = (ntiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
  p.scores = scores;
  p.hist = hist;
  p.bmax = bmax;
  p.bhist = bhist;
  p.nb = nb;
  p.block_len = a->pool_block_len;
  p.q_early = q_early ? 1 : 0;
  static SmemAttrOnce attr;
  const cudaError_t ea = attr.set(index_score_mx_kernel, kMxSmemBytes);
  if (ea != cudaSuccess) return ea;
  ProfScope ps(stream, "index_score_mx");
  launch_k(index_score_mx_kernel, dim3((unsigned)ctas_row, (unsigned)a->B), dim3(kMxThreads), kMxSmemBytes, stream,
           map, p);
  note_launches(1);
  return cudaGetLastError();
}

int read_mx_error(bool clear) {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_mx_error, sizeof(int));
  if (clear && v) {
    int z = 0;
    cudaMemcpyToSymbol(g_mx_error, &z, sizeof(int));
  }
  return v;
}

}  // namespace csa
