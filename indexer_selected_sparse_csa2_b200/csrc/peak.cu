// Measurement kernels: the denominators of the roofline fractions, measured
// in the same run as the kernels they judge (the pages report no hardware
// figure, so these have no counterpart there).
//
//   copy_peak_kernel  128-bit vectorised device-to-device copy (HBM peak:
//                     read + write bytes over time);
//   fp8_gemm_kernel   dense E4M3 x E4M3 -> fp32 GEMM D = A * B^T on the
//                     5th-generation tensor cores (FP8 dense peak): a
//                     persistent, warp-specialised tcgen05 kernel.
//                     warp 0  TMA producer: per stage a 128 x 128-byte A tile
//                             and a 256 x 128-byte B tile (128-byte swizzle),
//                             4-stage ring;
//                     warp 1  MMA issuer: 4 x tcgen05.mma kind::f8f6f4
//                             (M = 128, N = 256, K = 32) per stage into one
//                             of two 256-column TMEM accumulators;
//                     warps 2-5  epilogue: tcgen05.ld of the finished
//                             accumulator, fp32 stores, while the issuer
//                             fills the other accumulator.
// All waits are bounded (sm100.cuh).
#include "sm100.cuh"

namespace csa {

// ------------------------------------------------------------------ copy --
constexpr int kCpUnroll = 8;                     // 16-byte loads in flight per thread
constexpr size_t kCpTile = 256 * kCpUnroll;      // uint4 per CTA tile (32 KB)

__global__ void __launch_bounds__(256) copy_peak_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                        size_t n16) {
  pdl_enter();
  // contiguous 32 KB tiles, grid-strided; each warp's 8 loads cover 8
  // consecutive 512-byte segments of its tile
  const size_t ntiles = n16 / kCpTile;
  for (size_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const size_t base = t * kCpTile + threadIdx.x;
    uint4 v[kCpUnroll];
#pragma unroll
    for (int k = 0; k < kCpUnroll; ++k) v[k] = ld_nc_v4(src + base + (size_t)k * 256);
#pragma unroll
    for (int k = 0; k < kCpUnroll; ++k) dst[base + (size_t)k * 256] = v[k];
  }
  // ragged tail (< one tile), by the first CTA
  if (blockIdx.x == 0)
    for (size_t i = ntiles * kCpTile + threadIdx.x; i < n16; i += blockDim.x) dst[i] = ld_nc_v4(src + i);
}

// -------------------------------------------------------------- FP8 GEMM --
constexpr int kGmM = 128;
constexpr int kGmN = 256;
constexpr int kGmKB = 128;                       // K bytes (= E4M3 elements) per stage
constexpr int kGmStages = 4;
constexpr int kGmABytes = kGmM * kGmKB;          // 16 KB
constexpr int kGmBBytes = kGmN * kGmKB;          // 32 KB
constexpr int kGmThreads = 192;
constexpr uint32_t kGmTmemCols = 512;            // two 256-column accumulators
constexpr size_t kGmSmemBytes = 1024 + (size_t)kGmStages * (kGmABytes + kGmBBytes) + 256;

static __device__ int g_pk_error;

__global__ void __launch_bounds__(kGmThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, float* D,
                int M, int N, int K) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sa = base;
  uint8_t* sb = base + (size_t)kGmStages * kGmABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sb + (size_t)kGmStages * kGmBBytes);
  uint64_t* full = bars;                  // [kGmStages] TMA -> MMA
  uint64_t* empty = bars + kGmStages;     // [kGmStages] MMA -> TMA
  uint64_t* accf = bars + 2 * kGmStages;  // [2] accumulator ready
  uint64_t* acce = accf + 2;              // [2] accumulator drained (4 epilogue warps)
  uint64_t* drain = acce + 2;             // every MMA retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = M / kGmM, tiles_n = N / kGmN, ntiles = tiles_m * tiles_n, kblocks = K / kGmKB;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGmStages; ++i) { mbar_init(full + i, 1); mbar_init(empty + i, 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(accf + i, 1); mbar_init(acce + i, 4); }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&ta);
    prefetch_tmap(&tb);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kGmTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int tm = tile % tiles_m, tn = tile / tiles_m;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % kGmStages, ph = (it / kGmStages) & 1u;
          if (!mbar_wait(empty + s, ph ^ 1u, &g_pk_error, kErrWaitSmemEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(full + s, kGmABytes + kGmBBytes);
          tma_load_2d(sa + (size_t)s * kGmABytes, &ta, full + s, kb * kGmKB, tm * kGmM);
          tma_load_2d(sb + (size_t)s * kGmBBytes, &tb, full + s, kb * kGmKB, tn * kGmN);
        }
      }
      drain_copies(full, kGmStages, it, &g_pk_error, kErrWaitTmaFull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_make(kFmtE4M3, kFmtE4M3, kGmM, kGmN);
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++t) {
        const uint32_t a = t & 1u;
        if (!mbar_wait(acce + a, ((t >> 1) & 1u) ^ 1u, &g_pk_error, kErrWaitAccEmpty)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tbase + a * (uint32_t)kGmN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % kGmStages, ph = (it / kGmStages) & 1u;
          if (!mbar_wait(full + s, ph, &g_pk_error, kErrWaitTmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_s = smem_u32(sa + (size_t)s * kGmABytes), b_s = smem_u32(sb + (size_t)s * kGmBBytes);
#pragma unroll
          for (int k = 0; k < kGmKB / 32; ++k)
            mma_f8f6f4_ss(d, desc_k_sw128(a_s + 32u * k), desc_k_sw128(b_s + 32u * k), idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(empty + s);
        }
        mma_commit(accf + a);
      }
      mma_commit(drain);
      mbar_wait(drain, 0u, &g_pk_error, kErrWaitAccFull);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31 (rows of the tile)
    const int q = warp & 3;
    uint32_t t = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++t) {
      const int tm = tile % tiles_m, tn = tile / tiles_m;
      const uint32_t a = t & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(accf + a, (t >> 1) & 1u, &g_pk_error, kErrWaitAccFull));
      if (!ok) break;
      tc_fence_after();
      const int64_t row = (int64_t)tm * kGmM + 32 * q + lane;
      float* drow = D + row * N + (int64_t)tn * kGmN;
#pragma unroll 1
      for (int c = 0; c < kGmN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + a * (uint32_t)kGmN + (uint32_t)c, r);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(drow + c + 4 * v) = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce + a);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kGmTmemCols);
  }
}

// ----------------------------------------------------------------- host --
typedef CUresult (*EncodeTiledFn2)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn2 encode_fn2() {
  static EncodeTiledFn2 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn2>(f);
  }
  return fn;
}

// Row-major [rows][K] bytes, box K 128 bytes x box_rows rows, 128-byte swizzle.
static bool make_rows_tmap(CUtensorMap* map, const uint8_t* p, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn2 fn = encode_fn2();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K};
  const cuuint32_t box[2] = {(cuuint32_t)kGmKB, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int read_pk_error(bool clear) {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_pk_error, sizeof(int));
  if (clear && v) {
    int z = 0;
    cudaMemcpyToSymbol(g_pk_error, &z, sizeof(int));
  }
  return v;
}

}  // namespace csa

using namespace csa;

extern "C" {

csa_status csa_bench_copy(const void* src, void* dst, size_t bytes, csa_stream_t stream) {
  if (!src || !dst) return CSA_ERR_INVALID_ARG;
  if ((bytes & 15) || ((uintptr_t)src & 15) || ((uintptr_t)dst & 15)) return CSA_ERR_ALIGNMENT;
  if (bytes == 0) return CSA_OK;
  const size_t n16 = bytes / 16;
  size_t g = (n16 + kCpTile - 1) / kCpTile;
  const size_t gmax = (size_t)kNumSMs * 8;        // 8 resident CTAs of 256 threads per SM
  if (g == 0) g = 1;
  if (g > gmax) g = gmax;
  cudaStream_t st = (cudaStream_t)stream;
  {
    ProfScope ps(st, "copy_peak");
    launch_k(copy_peak_kernel, dim3((unsigned)g), dim3(256), 0, st, static_cast<const uint4*>(src),
             static_cast<uint4*>(dst), n16);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

csa_status csa_bench_fp8_gemm(const uint8_t* A, const uint8_t* B, float* D, int32_t M, int32_t N, int32_t K,
                              csa_stream_t stream) {
  if (!A || !B || !D) return CSA_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M % kGmM || N % kGmN || K % kGmKB) return CSA_ERR_SHAPE;
  if (((uintptr_t)A & 15) || ((uintptr_t)B & 15) || ((uintptr_t)D & 15)) return CSA_ERR_ALIGNMENT;
  CUtensorMap ma, mb;
  if (!make_rows_tmap(&ma, A, M, K, kGmM) || !make_rows_tmap(&mb, B, N, K, kGmN)) return CSA_ERR_CUDA;
  static SmemAttrOnce attr;
  if (attr.set(fp8_gemm_kernel, kGmSmemBytes) != cudaSuccess) return CSA_ERR_CUDA;
  const int ntiles = (M / kGmM) * (N / kGmN);
  const int grid = ntiles < kNumSMs ? ntiles : kNumSMs;
  cudaStream_t st = (cudaStream_t)stream;
  {
    ProfScope ps(st, "fp8_gemm_peak");
    launch_k(fp8_gemm_kernel, dim3(grid), dim3(kGmThreads), kGmSmemBytes, st, ma, mb, D, M, N, K);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // extern "C"
