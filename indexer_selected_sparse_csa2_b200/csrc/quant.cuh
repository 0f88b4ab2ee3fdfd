// Batched cache-entry encoding (the appends of a layer stack in one launch).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace csa {

constexpr int kMaxBatchJobs = 24;
// Batch job format (besides the csa_kv_format values): stage a token's 64-head
// attention query for the tcgen05 attention kernel (q2.cuh); n_rows = tokens
// x 64 heads, src = fp32 queries [tokens][64][512], dst = [tokens][128 KB].
constexpr int kFmtStageQ2 = 1000;

struct QuantBatchJob {
  const void* src;
  int64_t n_rows;
  int64_t src_stride_bytes;
  uint8_t* dst;
  int64_t dst_stride;
  int fmt;                 // csa_kv_format
  int bf16;                // source is bf16 (else fp32)
  int dim;
  int64_t unit0;           // first warp unit of this job in the flat list
  const float* aux;        // query staging: optional [tokens][32][2] RoPE (cos, sin) table
};

struct QuantBatch {
  QuantBatchJob job[kMaxBatchJobs];
  int njobs;
  int64_t units;           // warp units of all jobs
  uint4* zero_ptr;         // optional range cleared by the same launch
  int64_t zero_n16;        // its size in 16-byte words
};

// Warp units a job of this format and shape takes.
int64_t quant_batch_units(int fmt, int64_t n_rows, int dim);
cudaError_t launch_quant_batch(const QuantBatch& qb, cudaStream_t stream);

}  // namespace csa
