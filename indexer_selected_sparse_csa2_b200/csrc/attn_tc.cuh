// Parameters of the tcgen05 sparse-attention kernel (64 heads), shared by its
// launcher (attn_tc.cu) and the dispatch in attn_mma.cu.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace csa {

struct AttnTcParams {
  int B, n_q;
  int H;                      // 16, 32 or 64 query heads (the kernel runs 64, rows past H are zero)
  const float* q;
  const uint8_t* kv;
  int64_t kv_row_stride, kv_batch_stride;
  const int32_t* idx;
  int K;
  const uint8_t* win;
  int64_t win_row_stride, win_batch_stride;
  int n_win;
  float scale_log2;
  const float* sink;
  float* out;
  float* lse;
  int n_entries;
  int tiles_per_split;        // in 64-entry tiles
  int n_splits;
  const uint8_t* q2;          // optional: q already staged (q2.cuh layout), [B*n_q] tokens
  float* part_o;              // [B*n_q][n_splits][64][512] when n_splits > 1
  float* part_ml;             // [B*n_q][n_splits][64][2]
  const float* rope_cs;       // optional [B*n_q][32][2] (cos, sin): partial RoPE of q, inverse on out
  int out_bf16;               // out is bf16
};

cudaError_t launch_attn_tc(const AttnTcParams& p, cudaStream_t stream);

}  // namespace csa
