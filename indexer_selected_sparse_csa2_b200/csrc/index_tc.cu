// Decode indexer scoring over all cached positions on the 5th-generation
// tensor cores (tcgen05), keys streamed by TMA.
//
// Same function as index_score_decode_kernel (lightning-indexer score
// S[s] = sum_j w[j] * relu(<qI[j], kI[s]>), Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row), built the
// sm_100a way:
//   warp 0  TMA producer: 128-position x 64-byte key tiles (8 KB, 64-byte
//           swizzle) into a 5-stage shared-memory ring;
//   warp 1  MMA issuer: per tile two tcgen05.mma kind::f8f6f4 (M = 128
//           positions, N = 16 query heads, K = 2 x 32 bytes), fp32
//           accumulators in TMEM, six accumulator buffers;
//   warps 2-13  epilogue, three groups of four warps taking tiles in turn
//           (one group alone is latency-bound): one thread per position
//           reads its 16 head dots
//           from TMEM (tcgen05.ld), applies ReLU and the head weights, stores
//           the fp32 score, adds it to the 4096-bin histogram of the Top-K
//           select and, when building the candidate pool, the block max.
// Inside a layer stack the scan overlaps the stack's prologue kernel (the
// appended rows and the cleared histograms): the kernel triggers at once, the
// producer loads key tiles below `safe_rows` (the first row the prologue
// writes) before waiting for the prologue, and only the histogram flush and
// the tiles from safe_rows on wait.  Scores and block maxima go to buffers
// the prologue does not touch.  All waits are bounded (see sm100.cuh).
#include "sm100.cuh"
#include "select.cuh"

namespace csa {

constexpr int kTcEpiGroups = 3;
constexpr int kTcThreads = 64 + 128 * kTcEpiGroups;
constexpr int kTcStages = 5;
constexpr int kTcAcc = 2 * kTcEpiGroups;
constexpr int kTcRows = 128;
constexpr int kTcN = 16;                              // heads per MMA (8 used, rest zero)
constexpr int kTcStageBytes = kTcRows * 64;           // 8 KB
constexpr uint32_t kTcTmemCols = 128;                 // >= kTcAcc * kTcN, power of two

static __device__ int g_tc_error;

struct TcScoreParams {
  const uint8_t* q;     // [B][H_I][64]
  const float* w;       // [B][H_I]
  int H_I;
  int64_t T;
  int tiles_per_cta;
  float* scores;        // [B][T]
  uint32_t* hist;       // [B][4096]
  float* bmax;          // optional [B][nb]
  uint32_t* bhist;      // [B][4096]
  int64_t nb;
  int block_len;
  int64_t safe_rows;    // rows below this may be read before the wait; < 0: wait first
};

struct TcSmem {
  uint8_t* stage;        // kTcStages x 8 KB, 1024-byte aligned
  uint8_t* qb;           // 16 x 64 B swizzled query rows
  uint32_t* h;           // 4096
  uint32_t* hb;          // 4096
  uint64_t* full;
  uint64_t* empty;
  uint64_t* accf;
  uint64_t* acce;
  uint32_t* tmem_base;
};

constexpr size_t kTcSmemBytes = 1024 /*align slack*/ + (size_t)kTcStages * kTcStageBytes + 1024 /*qb*/ +
                                2 * kHistBins * 4 + 2 * (kTcStages + kTcAcc) * 8 + 16;

CSA_DEV TcSmem carve_tc_smem(uint8_t* raw) {
  TcSmem s;
  uintptr_t base = (reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  s.stage = p; p += (size_t)kTcStages * kTcStageBytes;
  s.qb = p; p += 1024;
  s.h = reinterpret_cast<uint32_t*>(p); p += kHistBins * 4;
  s.hb = reinterpret_cast<uint32_t*>(p); p += kHistBins * 4;
  s.full = reinterpret_cast<uint64_t*>(p); p += kTcStages * 8;
  s.empty = reinterpret_cast<uint64_t*>(p); p += kTcStages * 8;
  s.accf = reinterpret_cast<uint64_t*>(p); p += kTcAcc * 8;
  s.acce = reinterpret_cast<uint64_t*>(p); p += kTcAcc * 8;
  s.tmem_base = reinterpret_cast<uint32_t*>(p);
  return s;
}

__global__ void __launch_bounds__(kTcThreads, 3)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcScoreParams p) {
  pdl_trigger();
  const bool pre = p.safe_rows >= 0;
  if (!pre) pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  TcSmem S = carve_tc_smem(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y;
  const int64_t ntiles_row = (p.T + kTcRows - 1) / kTcRows;
  const int64_t tile0 = (int64_t)blockIdx.x * p.tiles_per_cta;
  const int64_t tile1 = min(tile0 + p.tiles_per_cta, ntiles_row);
  const int n_my = tile1 > tile0 ? (int)(tile1 - tile0) : 0;
  const bool build = p.bmax != nullptr;

  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < kTcAcc; ++i) { mbar_init(&S.accf[i], 1); mbar_init(&S.acce[i], 4); }
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  for (int i = tid; i < kHistBins; i += kTcThreads) { S.h[i] = 0; S.hb[i] = 0; }
  // query heads as the B operand: 16 rows x 64 bytes, 64-byte swizzle, zero rows past H_I
  for (int i = tid; i < kTcN * 64; i += kTcThreads) {
    const int r = i >> 6, c = i & 63;
    const uint8_t v = r < p.H_I ? p.q[((int64_t)b * p.H_I + r) * kDI + c] : (uint8_t)0;
    S.qb[sw64_offset(r, c)] = v;
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(S.tmem_base, kTcTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *S.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      bool waited = !pre;
      int issued = 0;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kTcStages;
        const uint32_t ph = (uint32_t)(i / kTcStages) & 1u;
        if (!waited && (tile0 + i + 1) * kTcRows > p.safe_rows) {
          pdl_wait();                 // this tile holds rows the prologue writes
          waited = true;
        }
        if (!mbar_wait(&S.empty[s], ph ^ 1u, &g_tc_error, kErrWaitSmemEmpty)) break;
        mbar_arrive_expect_tx(&S.full[s], kTcStageBytes);
        tma_load_3d(S.stage + (size_t)s * kTcStageBytes, &tmap, &S.full[s], 0, (int)((tile0 + i) * kTcRows), b);
        issued = i + 1;
      }
      drain_copies(S.full, kTcStages, issued, &g_tc_error, kErrWaitTmaFull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_make(kFmtE4M3, kFmtE4M3, kTcRows, kTcN);
      const uint64_t bdesc = desc_k_sw64(smem_u32(S.qb));
      for (int i = 0; i < n_my; ++i) {
        const int s = i % kTcStages, a = i % kTcAcc;
        if (!mbar_wait(&S.full[s], (uint32_t)(i / kTcStages) & 1u, &g_tc_error, kErrWaitTmaFull)) break;
        if (!mbar_wait(&S.acce[a], ((uint32_t)(i / kTcAcc) & 1u) ^ 1u, &g_tc_error, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint64_t adesc = desc_k_sw64(smem_u32(S.stage + (size_t)s * kTcStageBytes));
        const uint32_t d = tbase + (uint32_t)(a * kTcN);
        mma_f8f6f4_ss(d, adesc, bdesc, idesc, 0u);
        mma_f8f6f4_ss(d, adesc + 2, bdesc + 2, idesc, 1u);    // K bytes 32..63 (+32 B start address)
        mma_commit(&S.empty[s]);
        mma_commit(&S.accf[a]);
      }
    }
  } else {
    // epilogue: group g takes tiles g, g + G, ...; warp w reads TMEM lanes
    // 32*(w%4) .. +31 = rows of the tile
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;
    float wj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) wj[j] = j < p.H_I ? p.w[(int64_t)b * p.H_I + j] : 0.f;
    float* sc = p.scores + (int64_t)b * p.T;
    const int bl = p.block_len;
    for (int i = grp; i < n_my; i += kTcEpiGroups) {
      const int a = i % kTcAcc;
      if (!mbar_wait(&S.accf[a], (uint32_t)(i / kTcAcc) & 1u, &g_tc_error, kErrWaitAccFull)) break;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tbase + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * kTcN), r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acce[a]);
      float t8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t8[j] = wj[j] * fmaxf(__uint_as_float(r[j]), 0.f);
      const float s = ((t8[0] + t8[1]) + (t8[2] + t8[3])) + ((t8[4] + t8[5]) + (t8[6] + t8[7]));
      const int64_t row = (tile0 + i) * kTcRows + 32 * quarter + lane;
      const bool valid = row < p.T;
      if (valid) {
        sc[row] = s;
        if (p.hist) atomicAdd(&S.h[order_key(s) >> (32 - kHistBits)], 1u);
      }
      if (build) {
        float m = valid ? s : -INFINITY;
        for (int o = 1; o < bl; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((lane % bl) == 0 && valid) {
          p.bmax[(int64_t)b * p.nb + row / bl] = m;
          atomicAdd(&S.hb[order_key(m) >> (32 - kHistBits)], 1u);
        }
      }
    }
  }
  __syncthreads();
  if (pre) pdl_wait();                    // the histograms were cleared by the prologue
  uint32_t* gh = p.hist ? p.hist + (int64_t)b * kHistBins : nullptr;
  uint32_t* gbh = build ? p.bhist + (int64_t)b * kHistBins : nullptr;
  for (int i = tid; i < kHistBins; i += kTcThreads) {
    if (gh && S.h[i]) atomicAdd(&gh[i], S.h[i]);
    if (build && S.hb[i]) atomicAdd(&gbh[i], S.hb[i]);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTcTmemCols);
  }
}

// ----------------------------------------------------------------- host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// Key tensor map: dims (64 bytes, T positions, B sequences), box 64 x 128 x 1.
bool make_key_tmap(CUtensorMap* map, const uint8_t* keys, int64_t T, int B, int64_t row_stride,
                   int64_t batch_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (batch_stride == 0) batch_stride = row_stride * T;
  const cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride, (cuuint64_t)batch_stride};
  const cuuint32_t box[3] = {64, kTcRows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(keys), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E2M1 key codes (64 bytes = 128 codes per key) for kind::f8f6f4 operands:
// the packed 4-bit type copies every 16 codes into a 16-byte slot (8 bytes of
// codes, 8 bytes left unwritten), 128-key x 128-code boxes, 128-byte swizzle.
// The type needs a 32-byte aligned base and 32-byte multiple strides.
bool make_key_tmap_e2m1(CUtensorMap* map, const uint8_t* keys, int64_t T, int B, int64_t row_stride,
                        int64_t batch_stride, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (batch_stride == 0) batch_stride = row_stride * T;
  const cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride, (cuuint64_t)batch_stride};
  const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<uint8_t*>(keys), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_score_tc(const csa_index_args* a, float* scores, uint32_t* hist, float* bmax, uint32_t* bhist,
                            int64_t nb, int64_t safe_rows, cudaStream_t stream) {
  CUtensorMap map;
  if (!make_key_tmap(&map, a->keys, a->T, a->B, a->key_row_stride, a->key_batch_stride))
    return cudaErrorInvalidValue;
  TcScoreParams p{};
  p.q = a->q;
  p.w = a->w;
  p.H_I = a->H_I;
  p.T = a->T;
  const int64_t ntiles = (a->T + kTcRows - 1) / kTcRows;
  // three resident CTAs per SM (about 75 KB of shared memory, 128 TMEM
  // columns and 40 registers a thread each): each CTA's copies land at a
  // bounded rate, so more CTAs per SM keep more of HBM busy (two: 154.5 us
  // per hier_1m step, three: 153.4 us)
  int64_t ctas_row = 3 * kNumSMs / a->B;                 // one wave (rounded down)
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
  p.safe_rows = safe_rows;
  static SmemAttrOnce attr;
  const cudaError_t ea = attr.set(index_score_tc_kernel, kTcSmemBytes);
  if (ea != cudaSuccess) return ea;
  ProfScope ps(stream, "index_score_tc[full]");
  launch_k(index_score_tc_kernel, dim3(dim3((unsigned)ctas_row, (unsigned)a->B)), dim3(kTcThreads), kTcSmemBytes, stream, map, p);
  note_launches(1);
  return cudaGetLastError();
}

int read_tc_error(bool clear) {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(int));
  if (clear && v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof(int));
  }
  return v;
}

}  // namespace csa
