// Exact Top-K selection over rows of fp32 values (declarations).
#pragma once
#include "common.cuh"

namespace csa {

// One selection problem over B rows: the K largest values of each row, ties
// broken towards the lower slot, written as ascending positions.
struct SelectJob {
  const float* vals;        // [B][row_stride] values (slot s of row b)
  int64_t row_stride;
  int64_t n;                // slots per row (upper bound)
  const int32_t* n_row;     // optional per-row slot count (<= n)
  uint32_t* hist;           // [B][kHistBins] counts of order_key >> 20 (filled before extract)
  int K;
  // candidate buffers (workspace)
  uint32_t* cand_key;       // [B][n]
  int32_t* cand_pos;        // [B][n]
  uint32_t* list_key;       // [B][n] ordered contiguous copy (used when the list exceeds smem)
  int32_t* list_pos;        // [B][n]
  int32_t* cnt;             // [B][nchunks] candidates found in each run
  int64_t chunk;            // slots per run (one warp of an extract CTA scans one run)
  int nchunks;              // runs per row (<= 8192)
  // output
  int32_t* out;             // [B][out_stride]
  int64_t out_stride;
  int32_t out_width;        // entries per output row (K, or K * expand)
  const int32_t* map;       // optional slot -> position map [B][map_stride]
  int64_t map_stride;
  int expand;               // 0: write slots; >0: write `expand` positions per selected slot
  int32_t* out_len;         // [B] valid positions written (expand mode)
  int64_t limit;            // expand mode: positions >= limit are dropped
};

struct SelectPlan {
  int64_t chunk;
  int nchunks;
};

SelectPlan plan_select(int B, int64_t n);
// Bytes of workspace one SelectJob needs (hist + candidate buffers + counts).
size_t select_workspace_bytes(int B, int64_t n);
// Carve a job's buffers from `ws` (aligned), returning bytes used.
size_t select_carve(SelectJob& j, int B, int64_t n, void* ws);

// Launch: [optional hist] -> extract -> final for up to two jobs sharing B.
cudaError_t launch_select(const SelectJob* jobs, int njobs, int B, bool build_hist,
                          cudaStream_t stream);
cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t stream);

// Selection on thread-block clusters (select_cluster.cu): one cluster per
// (row, job), no workspace beyond the histogram given for rows read from memory.
struct CsRow {
  const float* vals;        // [B][row_stride] values (rows read from memory)
  int64_t row_stride;       // also the row stride of the fused pool variant's score output
  int vec;                  // vals 16-byte aligned and row_stride a multiple of 4
  int64_t n;                // slots per row (upper bound)
  const int32_t* n_row;     // optional per-row slot count (<= n)
  const uint32_t* hist;     // [B][kHistBins] counts of order_key >> 20 (rows read from memory)
  int K;
  int32_t* out;
  int64_t out_stride;
  int32_t out_width;
  const int32_t* map;       // optional slot -> position map (the pool, for pool rows)
  int64_t map_stride;
  int expand;
  int32_t* out_len;
  int64_t limit;
  int64_t run;              // slots per warp: cs_run(n)
};
struct CsJobs {
  CsRow j[2];
};
// Front-end of the pool-row variants: the values of the pool's slots are
// computed here (keys, q, w) or, with gscores, gathered from a score row.
struct CsPool {
  const uint8_t* keys;
  int64_t key_row_stride;
  int64_t key_batch_stride;
  const uint8_t* q;         // [B][H_I][64] E4M3
  const float* w;           // [B][H_I]
  int H_I;
  const int32_t* pool_len;  // [B]
  float* scores;            // optional [B][row_stride] score output
  const float* gscores;     // gather variant: scores [B][gscore_stride] by position
  int64_t gscore_stride;
};
int64_t cs_run(int64_t n);
bool cs_pool_ok(int64_t pool_cap);
cudaError_t launch_cluster_select(const CsRow* rows, int njobs, int B, cudaStream_t stream, const char* name);
cudaError_t launch_cluster_pool_select(const CsRow& row, const CsPool& pp, int B, cudaStream_t stream);
// First-level histograms of `B` rows of values (hist must be zeroed).
cudaError_t launch_hist_only(const float* vals, int64_t row_stride, int64_t n, const int32_t* n_row,
                             uint32_t* hist, int B, cudaStream_t stream);

}  // namespace csa
