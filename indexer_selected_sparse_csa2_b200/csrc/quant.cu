// Cache-entry encoders: FP4 main KV, FP8 windowed KV, plain E4M3 cast.
//
// FP4 main-KV entry (DeepSeek-V4.1 blog, "DeepSeek-V4.1-Flash" section, CSA2
// paragraph: E2M1 with one E4M3 scale per 16 channels; DeepSeek-V4.1-Flash
// architecture database, storage of the main-KV groups: 256 data bytes + 32
// float8_e4m3 scale bytes).  FP8 window entry (same database, storage of the
// "SWA window" group: E4M3 data with E8M0 scales per 32 channels, 512 + 16
// bytes).  Scale rules: see csa_kv_format in csa.h.
//
// One warp encodes one 512-channel row; lane l owns channels [16l, 16l+16),
// i.e. exactly one FP4 scale block, or half of one FP8 scale block.  Rows are
// read and written with 128-bit accesses (FP4 codes and scales gathered across
// lanes by shuffles).
#include "common.cuh"
#include "quant.cuh"
#include "q2.cuh"

namespace csa {

template <int SRC>  // 0 = fp32, 1 = bf16
CSA_DEV void load16(const void* row, int lane, float (&x)[16]) {
  if (SRC == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(row) + 16 * lane);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 v = ld_nc_v4(p + i);
      x[4 * i + 0] = __uint_as_float(v.x);
      x[4 * i + 1] = __uint_as_float(v.y);
      x[4 * i + 2] = __uint_as_float(v.z);
      x[4 * i + 3] = __uint_as_float(v.w);
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(row) + 16 * lane);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint4 v = ld_nc_v4(p + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[8 * i + 2 * k + 0] = __uint_as_float(w[k] << 16);          // bf16 -> fp32 is exact
        x[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
      }
    }
  }
}

// Lane `lane` of a warp encodes channels [16 lane, 16 lane + 16) of one FP4
// entry (one scale block) from values in registers.  Called by all 32 lanes
// of a warp for one entry: the entry is written with 16-byte stores (each
// even lane stores its codes and its odd neighbour's, lanes 0 and 16 the 32
// scale bytes).
CSA_DEV void encode_fp4_vals(const float (&x)[16], int lane, uint8_t* out) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t s_code = enc_e4m3x2(0.f, __fdiv_rn(amax, 6.0f)) & 0xFF;
  const float s = dec_e4m3(s_code);
  uint32_t packed[2] = {0u, 0u};
  if (s != 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // even channel in the low nibble
      uint32_t b = enc_e2m1x2(__fdiv_rn(x[2 * i + 1], s), __fdiv_rn(x[2 * i], s));
      packed[i >> 2] |= b << (8 * (i & 3));
    }
  }
  const uint32_t n0 = __shfl_xor_sync(0xffffffffu, packed[0], 1);
  const uint32_t n1 = __shfl_xor_sync(0xffffffffu, packed[1], 1);
  if ((lane & 1) == 0) *reinterpret_cast<uint4*>(out + 8 * lane) = make_uint4(packed[0], packed[1], n0, n1);
  // scale bytes: lane 4w gathers the word of lanes 4w .. 4w + 3, then lanes
  // 0 and 16 gather four words each
  uint32_t word = s_code;
  word |= __shfl_down_sync(0xffffffffu, s_code, 1) << 8;
  word |= __shfl_down_sync(0xffffffffu, s_code, 2) << 16;
  word |= __shfl_down_sync(0xffffffffu, s_code, 3) << 24;
  uint32_t w4[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w4[k] = __shfl_sync(0xffffffffu, word, (lane & 16) + 4 * k);
  if ((lane & 15) == 0) *reinterpret_cast<uint4*>(out + 256 + lane) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

// One warp encodes row `row` of the source into one FP4 entry.
template <int SRC>
CSA_DEV void encode_fp4_row(const void* row, int lane, uint8_t* out) {
  float x[16];
  load16<SRC>(row, lane, x);
  encode_fp4_vals(x, lane, out);
}

template <int SRC>
__global__ void __launch_bounds__(256) quant_fp4_kernel(const void* __restrict__ src, int64_t n_rows,
                                                        int64_t src_stride_bytes,
                                                        uint8_t* __restrict__ dst, int64_t dst_stride) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows; r += warps)
    encode_fp4_row<SRC>(static_cast<const uint8_t*>(src) + r * src_stride_bytes, lane, dst + r * dst_stride);
}

// Smallest e with amax <= 448 * 2^e, clamped to [-127, 127]; amax == 0 -> -127.
// amax = (1 + m / 2^23) * 2^E for a normal fp32; 448 = 1.75 * 2^8, so the
// answer is E - 8 when the significand is at most 1.75 and E - 7 otherwise.
CSA_DEV int ue8m0_exponent(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int ef = (int)((u >> 23) & 0xFF);
  if (ef == 0) return -127;  // zero or subnormal: far below 448 * 2^-127
  const uint32_t m = u & 0x7FFFFFu;
  int e = (ef - 127) - 8 + (m > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^k as an fp32 value for k in [-127, 127] (2^-127 is subnormal).
CSA_DEV float pow2f(int k) {
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << 22);
}

// One warp encodes one row into one FP8 window entry.
template <int SRC>
CSA_DEV void encode_fp8w_row(const void* row, int lane, uint8_t* out) {
  float x[16];
  load16<SRC>(row, lane, x);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // 32-channel block = lane pair
  const int e = ue8m0_exponent(amax);
  const float sc = pow2f(-e);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo = enc_e4m3x2(x[4 * i + 1] * sc, x[4 * i + 0] * sc);
    uint32_t hi = enc_e4m3x2(x[4 * i + 3] * sc, x[4 * i + 2] * sc);
    w[i] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(out + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  if ((lane & 1) == 0) out[512 + (lane >> 1)] = (uint8_t)(e + 127);
}

template <int SRC>
__global__ void __launch_bounds__(256) quant_fp8w_kernel(const void* __restrict__ src, int64_t n_rows,
                                                         int64_t src_stride_bytes,
                                                         uint8_t* __restrict__ dst, int64_t dst_stride) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows; r += warps)
    encode_fp8w_row<SRC>(static_cast<const uint8_t*>(src) + r * src_stride_bytes, lane, dst + r * dst_stride);
}

// Plain E4M3 cast of 16 values in registers into column group c of a row.
CSA_DEV void encode_plain_vals(const float (&x)[16], int c, uint8_t* out_row) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo = enc_e4m3x2(x[4 * i + 1], x[4 * i + 0]);
    uint32_t hi = enc_e4m3x2(x[4 * i + 3], x[4 * i + 2]);
    w[i] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(out_row + 16 * c) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Plain E4M3 cast of 16 consecutive values (column group c of a row).
template <int SRC>
CSA_DEV void encode_plain16(const void* row, int c, uint8_t* out_row) {
  float x[16];
  // reuse the 16-value loader with "lane" = column group
  load16<SRC>(row, c, x);
  encode_plain_vals(x, c, out_row);
}

// ------------------------------------------------------------ compressor --
// The m-token compressor of the encoder's CSA2 layers (DeepSeek-V4.1-Flash
// architecture database, cache groups: one shared K=V entry per 2 tokens for
// the encoder's main KV and indexer K, pooled with a gate in fp32; the
// ratio-1 compressor is plain).  Per channel of a group of m token rows x_i
// with gate logits g_i: w_i = exp(g_i - max_j g_j), entry = sum_i w_i x_i /
// sum_i w_i, in fp32; then the entry is encoded like any cache row.  One
// thread = 16 channels of one group (one FP4 scale block); token row r of
// the source at src + r * src_stride_bytes, its gates at gate + r * gate_stride.
template <int SRC>
__global__ void __launch_bounds__(256) compress_kernel(const void* __restrict__ src, const float* __restrict__ gate,
                                                       int64_t n_groups, int m, int dim, int64_t src_stride_bytes,
                                                       int64_t gate_stride, int fmt, uint8_t* __restrict__ dst,
                                                       int64_t dst_stride) {
  pdl_enter();
  const int per_row = dim >> 4;
  const int64_t units = n_groups * per_row;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = u / per_row;
    const int c = (int)(u - n * per_row);
    float x[16];
    if (m == 1) {
      load16<SRC>(static_cast<const uint8_t*>(src) + n * src_stride_bytes, c, x);
    } else {
      float gmax[16], acc[16], wsum[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) { gmax[k] = -INFINITY; acc[k] = 0.f; wsum[k] = 0.f; }
      for (int i = 0; i < m; ++i) {
        const float4* gp = reinterpret_cast<const float4*>(gate + (n * m + i) * gate_stride + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 g = gp[q];
          gmax[4 * q] = fmaxf(gmax[4 * q], g.x); gmax[4 * q + 1] = fmaxf(gmax[4 * q + 1], g.y);
          gmax[4 * q + 2] = fmaxf(gmax[4 * q + 2], g.z); gmax[4 * q + 3] = fmaxf(gmax[4 * q + 3], g.w);
        }
      }
      for (int i = 0; i < m; ++i) {
        float xi[16];
        load16<SRC>(static_cast<const uint8_t*>(src) + (n * m + i) * src_stride_bytes, c, xi);
        const float4* gp = reinterpret_cast<const float4*>(gate + (n * m + i) * gate_stride + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 g = gp[q];
          const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float w = expf(gg[k] - gmax[4 * q + k]);
            acc[4 * q + k] = fmaf(w, xi[4 * q + k], acc[4 * q + k]);
            wsum[4 * q + k] += w;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) x[k] = __fdiv_rn(acc[k], wsum[k]);
    }
    if (fmt == CSA_FMT_FP4_E2M1_E4M3X16) encode_fp4_vals(x, c, dst + n * dst_stride);
    else encode_plain_vals(x, c, dst + n * dst_stride);
  }
}

cudaError_t launch_compress(const void* src, int src_dtype, const float* gate, int64_t n_groups, int m, int dim,
                            int64_t src_row_stride, int64_t gate_row_stride, int fmt, void* dst,
                            int64_t dst_row_stride, cudaStream_t stream) {
  const int64_t esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  const int64_t units = n_groups * (dim >> 4);
  int64_t g = (units + 255) / 256;
  if (g > kNumSMs * 8) g = kNumSMs * 8;
  if (g < 1) g = 1;
  // a group's rows are m consecutive token rows of src_row_stride elements
  const int64_t stride_b = src_row_stride * esz;
  ProfScope ps(stream, "compress");
  if (src_dtype == CSA_SRC_BF16)
    launch_k(compress_kernel<1>, dim3((unsigned)g), dim3(256), 0, stream, src, gate, n_groups, m, dim, stride_b,
             gate_row_stride, fmt, static_cast<uint8_t*>(dst), dst_row_stride);
  else
    launch_k(compress_kernel<0>, dim3((unsigned)g), dim3(256), 0, stream, src, gate, n_groups, m, dim, stride_b,
             gate_row_stride, fmt, static_cast<uint8_t*>(dst), dst_row_stride);
  note_launches(1);
  return cudaGetLastError();
}

// Plain E4M3 cast: each thread encodes 16 consecutive values of one row.
template <int SRC>
__global__ void __launch_bounds__(256) quant_plain_kernel(const void* __restrict__ src, int64_t n_rows,
                                                          int dim, int64_t src_stride_bytes,
                                                          uint8_t* __restrict__ dst, int64_t dst_stride) {
  pdl_enter();
  const int per_row = dim >> 4;
  const int64_t total = n_rows * per_row;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = g / per_row;
    const int c = (int)(g - r * per_row);
    encode_plain16<SRC>(static_cast<const uint8_t*>(src) + r * src_stride_bytes, c, dst + r * dst_stride);
  }
}

// ------------------------------------------------------------ batched jobs --
// All the appends of a layer stack (and the clearing of its histogram
// region) in one launch: a flat list of warp-sized units.  FP4 / FP8 rows
// are one unit per row; plain casts pack 32 groups of 16 values per unit;
// the zero range is 512 bytes per unit.
__global__ void __launch_bounds__(256) quant_batch_kernel(QuantBatch qb) {
  // wait, then trigger: a kernel after this one may start before it ends
  // (the stack's full scan reads the key rows this batch does not write), but
  // never before the work ahead of this batch on the stream has completed
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t zero_units = (qb.zero_n16 + 31) / 32;
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < qb.units + zero_units;
       u += warps) {
    if (u >= qb.units) {
      const int64_t i = (u - qb.units) * 32 + lane;
      if (i < qb.zero_n16) qb.zero_ptr[i] = make_uint4(0, 0, 0, 0);
      continue;
    }
    int j = 0;
    while (j + 1 < qb.njobs && u >= qb.job[j + 1].unit0) ++j;
    const QuantBatchJob& J = qb.job[j];
    const int64_t lu = u - J.unit0;
    const uint8_t* src = static_cast<const uint8_t*>(J.src);
    if (J.fmt == CSA_FMT_FP4_E2M1_E4M3X16) {
      if (J.bf16) encode_fp4_row<1>(src + lu * J.src_stride_bytes, lane, J.dst + lu * J.dst_stride);
      else encode_fp4_row<0>(src + lu * J.src_stride_bytes, lane, J.dst + lu * J.dst_stride);
    } else if (J.fmt == CSA_FMT_FP8_E4M3_UE8M0X32) {
      if (J.bf16) encode_fp8w_row<1>(src + lu * J.src_stride_bytes, lane, J.dst + lu * J.dst_stride);
      else encode_fp8w_row<0>(src + lu * J.src_stride_bytes, lane, J.dst + lu * J.dst_stride);
    } else if (J.fmt == kFmtStageQ2) {
      const int64_t tok = lu >> 6;
      encode_q2_head(reinterpret_cast<const float*>(src) + tok * (64 * 512), (int)(lu & 63), lane,
                     J.dst + tok * kQ2TokenBytes, J.aux ? J.aux + tok * 64 : nullptr);
    } else {
      const int per_row = J.dim >> 4;
      const int64_t g = lu * 32 + lane;
      if (g < J.n_rows * per_row) {
        const int64_t r = g / per_row;
        const int c = (int)(g - r * per_row);
        if (J.bf16) encode_plain16<1>(src + r * J.src_stride_bytes, c, J.dst + r * J.dst_stride);
        else encode_plain16<0>(src + r * J.src_stride_bytes, c, J.dst + r * J.dst_stride);
      }
    }
  }
}

int64_t quant_batch_units(int fmt, int64_t n_rows, int dim) {
  if (fmt == CSA_FMT_FP8_E4M3_PLAIN) return (n_rows * (dim >> 4) + 31) / 32;
  return n_rows;
}

cudaError_t launch_quant_batch(const QuantBatch& qb, cudaStream_t stream) {
  const int64_t units = qb.units + (qb.zero_n16 + 31) / 32;
  if (units == 0) return cudaSuccess;
  int64_t g = (units + 7) / 8;
  if (g > (int64_t)kNumSMs * 8) g = (int64_t)kNumSMs * 8;
  ProfScope ps(stream, "quant_batch");
  launch_k(quant_batch_kernel, dim3((unsigned)g), dim3(256), 0, stream, qb);
  note_launches(1);
  return cudaGetLastError();
}

static int grid_for(int64_t work, int per_block) {
  int64_t g = (work + per_block - 1) / per_block;
  const int64_t cap = (int64_t)kNumSMs * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

// ------------------------------------------------------------------ MXFP4 --
// MXFP4 indexer keys (DeepSeek-V4.1-Flash architecture database, storage of
// the indexer K groups: 4-bit E2M1 elements with one E8M0 scale per 32
// channels, 68 bytes per 128-channel entry).  Per block of 32 channels: e is
// the smallest integer with amax <= 6 * 2^e, clamped to [-127, 127] (amax = 0
// -> -127), and code_i = E2M1_rne_sat(x_i * 2^-e) (an exact power-of-two
// scaling unless the product underflows, where E2M1 gives +-0 anyway).  Codes
// go to a code plane (two per byte, even channel in the low nibble), the
// exponent bytes (e + 127) to a scale plane.
// 6 = 1.5 * 2^2: for amax = f * 2^E with f in [1, 2), e = E - 2 when f <= 1.5
// and E - 1 otherwise.
CSA_DEV int mx_exponent(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int ef = (int)((u >> 23) & 0xFF);
  if (ef == 0) return -127;  // zero or subnormal: 6 * 2^-127 >= amax
  const uint32_t m = u & 0x7FFFFFu;
  const int e = (ef - 127) - 2 + (m > 0x400000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// One thread encodes 32 channels (one scale block) of one row.
template <int SRC>
__global__ void __launch_bounds__(256) quant_mx_kernel(const void* __restrict__ src, int64_t n_rows, int dim,
                                                       int64_t src_stride_bytes, uint8_t* __restrict__ codes,
                                                       int64_t codes_stride, uint8_t* __restrict__ scales,
                                                       int64_t scales_stride) {
  pdl_enter();
  const int per_row = dim >> 5;
  const int64_t total = n_rows * per_row;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = g / per_row;
    const int blk = (int)(g - r * per_row);
    const uint8_t* row = static_cast<const uint8_t*>(src) + r * src_stride_bytes;
    float x[32];
    load16<SRC>(row, 2 * blk, *reinterpret_cast<float(*)[16]>(x));
    load16<SRC>(row, 2 * blk + 1, *reinterpret_cast<float(*)[16]>(x + 16));
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const int e = mx_exponent(amax);
    const float sc = pow2f(-e);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // even channel in the low nibble
      const uint32_t b = enc_e2m1x2(x[2 * i + 1] * sc, x[2 * i] * sc);
      w[i >> 2] |= b << (8 * (i & 3));
    }
    *reinterpret_cast<uint4*>(codes + r * codes_stride + 16 * blk) = make_uint4(w[0], w[1], w[2], w[3]);
    scales[r * scales_stride + blk] = (uint8_t)(e + 127);
  }
}

cudaError_t launch_quant_mx(const void* src, int src_dtype, int64_t n_rows, int dim, int64_t src_row_stride,
                            uint8_t* codes, int64_t codes_row_stride, uint8_t* scales, int64_t scales_row_stride,
                            cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const int esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  const int g = grid_for(n_rows * (dim / 32), 256);
  ProfScope ps(stream, "quant_mxfp4");
  if (src_dtype == CSA_SRC_F32)
    launch_k(quant_mx_kernel<0>, dim3(g), dim3(256), 0, stream, src, n_rows, dim, src_row_stride * esz, codes,
             codes_row_stride, scales, scales_row_stride);
  else
    launch_k(quant_mx_kernel<1>, dim3(g), dim3(256), 0, stream, src, n_rows, dim, src_row_stride * esz, codes,
             codes_row_stride, scales, scales_row_stride);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_quant(const void* src, int src_dtype, int64_t n_rows, int dim, int64_t src_row_stride,
                         int fmt, void* dst, int64_t dst_row_stride, cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const int esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  const int64_t sstride = src_row_stride * esz;
  uint8_t* d = static_cast<uint8_t*>(dst);
  ProfScope ps(stream, fmt == CSA_FMT_FP4_E2M1_E4M3X16 ? "quant_fp4" : (fmt == CSA_FMT_FP8_E4M3_UE8M0X32 ? "quant_fp8w" : "quant_plain"));
  if (fmt == CSA_FMT_FP4_E2M1_E4M3X16) {
    const int g = grid_for(n_rows, 8);
    if (src_dtype == CSA_SRC_F32) launch_k(quant_fp4_kernel<0>, dim3(g), dim3(256), 0, stream, src, n_rows, sstride, d, dst_row_stride);
    else launch_k(quant_fp4_kernel<1>, dim3(g), dim3(256), 0, stream, src, n_rows, sstride, d, dst_row_stride);
  } else if (fmt == CSA_FMT_FP8_E4M3_UE8M0X32) {
    const int g = grid_for(n_rows, 8);
    if (src_dtype == CSA_SRC_F32) launch_k(quant_fp8w_kernel<0>, dim3(g), dim3(256), 0, stream, src, n_rows, sstride, d, dst_row_stride);
    else launch_k(quant_fp8w_kernel<1>, dim3(g), dim3(256), 0, stream, src, n_rows, sstride, d, dst_row_stride);
  } else {
    const int g = grid_for(n_rows * (dim / 16), 256);
    if (src_dtype == CSA_SRC_F32) launch_k(quant_plain_kernel<0>, dim3(g), dim3(256), 0, stream, src, n_rows, dim, sstride, d, dst_row_stride);
    else launch_k(quant_plain_kernel<1>, dim3(g), dim3(256), 0, stream, src, n_rows, dim, sstride, d, dst_row_stride);
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace csa
