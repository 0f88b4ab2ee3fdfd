// Lightning-indexer scores over MXFP4 indexer keys on the tcgen05 tensor
// cores: the pages' production indexer (Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row: 32 heads of
// dimension 128; DeepSeek-V4.1-Flash architecture database, indexer K
// storage: E2M1 elements with one E8M0 scale per 32 channels, 68 bytes per
// entry), with plain E4M3 queries.
//   S[s] = sum_j w[j] * relu( sum_b 2^(e[s,b]) * <q[j, block b], k[s, block b]> )
// where k is the key's E2M1 codes and e its block exponents.
// Keys sit in two planes: codes [B][T][64 B] and exponent bytes [B][T][4].
//   warp 0     TMA producer: 128-key x 64-byte code tiles (64-byte swizzle)
//              into a 12-stage ring (96 KB in flight: one CTA per SM);
//   warp 1     MMA issuer: per tile, one tcgen05.mma kind::f8f6f4 per 32-channel
//              block (M = 128 keys, N = 32 heads, K = 32) into its own TMEM
//              accumulator (4 x 32 columns per tile, four tiles in flight);
//   warps 2-9  decode: two threads per key (64 channels each), E2M1 codes ->
//              E4M3 bytes (every E2M1 value is an E4M3 value) into a
//              128-byte-swizzled K-major tile, four tiles in flight;
//   warps 10-13 epilogue: one key per thread, the 4 x 32 block dots from TMEM,
//              times 2^e per block, ReLU, head weights, the fp32 score, the
//              first-level Top-K histogram and, when building the pool, the
//              block maxima.
// All waits are bounded (sm100.cuh).
#include "sm100.cuh"
#include "select.cuh"

namespace csa {

constexpr int kMxRows = 128;                    // keys per tile
constexpr int kMxHeads = 32;
constexpr int kMxStages = 12;                 // 96 KB of key tiles in flight per SM
constexpr int kMxStageBytes = kMxRows * 64;     // packed codes, 8 KB
constexpr int kMxDec = 4;                       // decoded tiles in flight
constexpr int kMxDecWarps = 8;
constexpr int kMxDecBytes = kMxRows * 128;      // 16 KB
constexpr int kMxEpiGroups = 1;
constexpr int kMxAcc = 4;
constexpr uint32_t kMxTmemCols = 128 * kMxAcc;  // kMxAcc x 4 blocks x 32 heads
constexpr int kMxEpiWarp0 = 2 + kMxDecWarps;
constexpr int kMxThreads = 32 * kMxEpiWarp0 + 128 * kMxEpiGroups;
constexpr size_t kMxSmemBytes = 1024 + (size_t)kMxStages * kMxStageBytes + (size_t)kMxDec * kMxDecBytes +
                                kMxHeads * 128 + 2 * kHistBins * 4 + 2 * (kMxStages + kMxDec + kMxAcc) * 8 + 16;

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
};

// E2M1 magnitude code -> E4M3 byte of the same value: 0, 0.5, 1, 1.5, 2, 3, 4, 6
constexpr uint32_t kE2M1toE4M3Lo = 0x3C383000u;
constexpr uint32_t kE2M1toE4M3Hi = 0x4C484440u;
// Four E2M1 codes (nibbles 0-3 of w) as four E4M3 bytes.
CSA_DEV uint32_t e2m1x4_to_e4m3(uint32_t w) {
  const uint32_t mag = __byte_perm(kE2M1toE4M3Lo, kE2M1toE4M3Hi, w & 0x7777u);
  const uint32_t sgn = ((w & 0x8u) << 4) | ((w & 0x80u) << 8) | ((w & 0x800u) << 12) | ((w & 0x8000u) << 16);
  return mag | sgn;
}

__global__ void __launch_bounds__(kMxThreads, 1)
index_score_mx_kernel(const __grid_constant__ CUtensorMap tmap, MxScoreParams p) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* stage = base;
  uint8_t* dec = stage + (size_t)kMxStages * kMxStageBytes;
  uint8_t* qb = dec + (size_t)kMxDec * kMxDecBytes;
  uint32_t* h = reinterpret_cast<uint32_t*>(qb + kMxHeads * 128);
  uint32_t* hb = h + kHistBins;
  uint64_t* bars = reinterpret_cast<uint64_t*>(hb + kHistBins);
  uint64_t* full = bars;                       // [kMxStages] TMA -> decode
  uint64_t* empty = full + kMxStages;          // [kMxStages] decode -> TMA (4 warps)
  uint64_t* dfull = empty + kMxStages;         // [kMxDec] decode -> MMA (4 warps)
  uint64_t* dempty = dfull + kMxDec;           // [kMxDec] MMA -> decode
  uint64_t* accf = dempty + kMxDec;            // [kMxAcc] MMA -> epilogue
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
    for (int i = 0; i < kMxStages; ++i) { mbar_init(full + i, 1); mbar_init(empty + i, kMxDecWarps); }
    for (int i = 0; i < kMxDec; ++i) { mbar_init(dfull + i, kMxDecWarps); mbar_init(dempty + i, 1); }
    for (int i = 0; i < kMxAcc; ++i) { mbar_init(accf + i, 1); mbar_init(acce + i, 4); }
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  for (int i = tid; i < kHistBins; i += kMxThreads) { h[i] = 0; hb[i] = 0; }
  // queries: the B operand, 32 rows of 128 bytes, 128-byte swizzle
  for (int i = tid; i < kMxHeads * 8; i += kMxThreads) {
    const int r = i >> 3, c = i & 7;
    const uint4 v = ld_v4(p.q + ((int64_t)b * kMxHeads + r) * 128 + 16 * c);
    *reinterpret_cast<uint4*>(qb + r * 128 + ((c ^ (r & 7)) << 4)) = v;
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_slot, kMxTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kMxStages;
        if (!mbar_wait(empty + s, ((uint32_t)(i / kMxStages) & 1u) ^ 1u, &g_mx_error, kErrWaitSmemEmpty)) break;
        mbar_arrive_expect_tx(full + s, kMxStageBytes);
        tma_load_3d(stage + (size_t)s * kMxStageBytes, &tmap, full + s, 0, (int)((tile0 + i) * kMxRows), b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_make(kFmtE4M3, kFmtE4M3, kMxRows, kMxHeads);
      const uint32_t qa = smem_u32(qb);
      for (int i = 0; i < n_my; ++i) {
        const int d = i % kMxDec, a = i % kMxAcc;
        if (!mbar_wait(dfull + d, (uint32_t)(i / kMxDec) & 1u, &g_mx_error, kErrWaitTmaFull)) break;
        if (!mbar_wait(acce + a, ((uint32_t)(i / kMxAcc) & 1u) ^ 1u, &g_mx_error, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t da = smem_u32(dec + (size_t)d * kMxDecBytes);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk)
          mma_f8f6f4_ss(tbase + (uint32_t)(a * 128 + 32 * blk), desc_k_sw128(da + 32u * blk),
                        desc_k_sw128(qa + 32u * blk), idesc, 0u);
        mma_commit(dempty + d);
        mma_commit(accf + a);
      }
    }
  } else if (warp < kMxEpiWarp0) {
    // ---- decode: threads 2r and 2r + 1 take key row r, packed chunks
    // {0, 1} and {2, 3} (64 channels each)
    const int r = (tid - 64) >> 1, hf = (tid - 64) & 1;
    for (int i = 0; i < n_my; ++i) {
      const int s = i % kMxStages, d = i % kMxDec;
      bool ok = __all_sync(0xffffffffu, mbar_wait(full + s, (uint32_t)(i / kMxStages) & 1u, &g_mx_error, kErrWaitTmaFull));
      if (i >= kMxDec)
        ok = ok && __all_sync(0xffffffffu, mbar_wait(dempty + d, ((uint32_t)(i / kMxDec) - 1u) & 1u, &g_mx_error,
                                                     kErrWaitSmemEmpty));
      if (!ok) break;
      const uint8_t* src = stage + (size_t)s * kMxStageBytes + r * 64;
      uint8_t* dst = dec + (size_t)d * kMxDecBytes + r * 128;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * hf + cc;
        // packed chunk c (channels 32c .. 32c + 31) at its 64-byte-swizzle position
        const uint4 v = *reinterpret_cast<const uint4*>(src + ((c ^ ((r >> 1) & 3)) << 4));
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {          // 16 channels -> one 16-byte chunk j = 2c + hh
          const uint32_t w0 = wv[2 * hh], w1 = wv[2 * hh + 1];
          const int j = 2 * c + hh;
          *reinterpret_cast<uint4*>(dst + ((j ^ (r & 7)) << 4)) =
              make_uint4(e2m1x4_to_e4m3(w0), e2m1x4_to_e4m3(w0 >> 16), e2m1x4_to_e4m3(w1), e2m1x4_to_e4m3(w1 >> 16));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) { mbar_arrive(empty + s); mbar_arrive(dfull + d); }
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

bool make_key_tmap(CUtensorMap* map, const uint8_t* keys, int64_t T, int B, int64_t row_stride,
                   int64_t batch_stride);

cudaError_t launch_score_mx(const csa_index_args* a, float* scores, uint32_t* hist, float* bmax, uint32_t* bhist,
                            int64_t nb, cudaStream_t stream) {
  CUtensorMap map;
  if (!make_key_tmap(&map, a->keys, a->T, a->B, a->key_row_stride, a->key_batch_stride)) return cudaErrorInvalidValue;
  MxScoreParams p{};
  p.q = a->q;
  p.w = a->w;
  p.scales = a->key_scales;
  p.scale_row_stride = a->key_scale_row_stride;
  p.scale_batch_stride = a->key_scale_batch_stride;
  p.T = a->T;
  const int64_t ntiles = (a->T + kMxRows - 1) / kMxRows;
  // one wave: at most one CTA per SM (rounded down, so that no CTA waits
  // for a second wave)
  int64_t ctas_row = kNumSMs / a->B;
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
