// Context-parallel decode of one long sequence: the cache positions [0, T)
// are split into contiguous shards, one per rank; each rank scores its own
// shard (csa_index_topk on the shard) and the ranks exchange small results.
// The pages give no multi-GPU scheme for this path; the exchange follows from
// the selection rule and the softmax (Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row: the K
// best-scored positions, ties to the lower position; "Multi-head latent
// attention" row: one softmax over the selected entries and the window):
//   - every entry of the global Top-K is among the K best of its own shard,
//     so the K best of the union of the shards' local Top-K lists, ranked by
//     (score descending, position ascending), is the global Top-K;
//   - per-rank attention over the selected entries a rank owns returns
//     (out_r, lse_r), and lse = log sum_r exp(lse_r),
//     out = sum_r exp(lse_r - lse) * out_r is one softmax over all entries.
// Kernels here: the local (score, position) pairs, the exact merge (a
// compaction, then the cluster Top-K over the rank-ordered candidates, whose
// slot order is position order), the localisation of the global Top-K to a
// shard, and the log-sum-exp combine.  The exchange itself (two all-gathers)
// is the caller's, e.g. NCCL.
#include "select.cuh"

namespace csa {

// (score, global position) of every local Top-K entry; padding -> (-inf, -1).
__global__ void cp_pairs_kernel(const int32_t* idx, const float* scores, int B, int K, int64_t score_stride,
                                int64_t t0, float* pair_score, int32_t* pair_pos) {
  pdl_enter();
  const int64_t n = (int64_t)B * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int b = (int)(i / K);
    const int32_t p = idx[i];
    pair_score[i] = p >= 0 ? scores[(int64_t)b * score_stride + p] : -INFINITY;
    pair_pos[i] = p >= 0 ? (int32_t)(p + t0) : -1;
  }
}

// Rank-ordered compaction of the gathered pairs [R][B][Kl] into one
// candidate row per sequence [B][R*Kl] (each rank's valid entries come first
// in its list, ascending, so the concatenation is ascending by position) and
// its length.  One CTA per sequence.
constexpr int kCpThreads = 256;
__global__ void __launch_bounds__(kCpThreads) cp_compact_kernel(const float* pair_score, const int32_t* pair_pos,
                                                               int R, int B, int Kl, float* c_score,
                                                               int32_t* c_pos, int32_t* c_len) {
  pdl_enter();
  const int b = blockIdx.x;
  __shared__ int32_t off[1025];
  // valid entries of each rank's list (a prefix of the list)
  for (int r = threadIdx.x; r < R; r += kCpThreads) {
    const int32_t* pp = pair_pos + ((int64_t)r * B + b) * Kl;
    int lo = 0, hi = Kl;                      // first index with pp < 0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pp[mid] >= 0) lo = mid + 1; else hi = mid;
    }
    off[r + 1] = lo;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    off[0] = 0;
    for (int r = 0; r < R; ++r) off[r + 1] += off[r];
    c_len[b] = off[R];
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    const int n = off[r + 1] - off[r];
    const float* ps = pair_score + ((int64_t)r * B + b) * Kl;
    const int32_t* pp = pair_pos + ((int64_t)r * B + b) * Kl;
    float* ds = c_score + (int64_t)b * R * Kl + off[r];
    int32_t* dp = c_pos + (int64_t)b * R * Kl + off[r];
    for (int i = threadIdx.x; i < n; i += kCpThreads) { ds[i] = ps[i]; dp[i] = pp[i]; }
  }
}

__global__ void cp_localize_kernel(const int32_t* idx, int64_t n, int64_t t0, int64_t t1, int32_t* idx_local) {
  pdl_enter();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t p = idx[i];
    idx_local[i] = (p >= t0 && p < t1) ? (int32_t)(p - t0) : -1;
  }
}

// out[b][h] = sum_r w_r o_r[b][h] / Z with w_r = exp(lse_r - M), M the max
// over ranks (and the sink), Z = sum_r w_r (+ exp(sink - M)); lse = M + log Z.
// One CTA per (sequence, head), 128 threads x 4 channels.
__global__ void __launch_bounds__(128) cp_combine_kernel(const float* o_parts, const float* lse_parts, int R, int B,
                                                         int H, const float* sink, float* out, float* lse) {
  pdl_enter();
  const int b = blockIdx.x, h = blockIdx.y;
  __shared__ float w_s[1024];
  __shared__ float inv_s;
  if (threadIdx.x < 32) {
    const float sk = sink ? sink[h] : -INFINITY;
    float M = sk;
    for (int r = threadIdx.x; r < R; r += 32) M = fmaxf(M, lse_parts[((int64_t)r * B + b) * H + h]);
    M = warp_max(M);
    float Z = 0.f;
    for (int r = threadIdx.x; r < R; r += 32) {
      const float l = lse_parts[((int64_t)r * B + b) * H + h];
      const float w = l == -INFINITY ? 0.f : expf(l - M);
      w_s[r] = w;
      Z += w;
    }
    Z = warp_sum(Z);
    if (threadIdx.x == 0) {
      if (sk != -INFINITY) Z += expf(sk - M);
      inv_s = Z > 0.f ? 1.f / Z : 0.f;
      if (lse) lse[(int64_t)b * H + h] = Z > 0.f ? M + logf(Z) : -INFINITY;
    }
  }
  __syncthreads();
  const int d = 4 * threadIdx.x;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < R; ++r) {
    const float w = w_s[r];
    if (w == 0.f) continue;
    const float4 v = *reinterpret_cast<const float4*>(o_parts + (((int64_t)r * B + b) * H + h) * kD + d);
    acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
  }
  const float inv = inv_s;
  *reinterpret_cast<float4*>(out + ((int64_t)b * H + h) * kD + d) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

static int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g < 1) g = 1;
  if (g > kNumSMs * 8) g = kNumSMs * 8;
  return (int)g;
}

}  // namespace csa

using namespace csa;

extern "C" {

csa_status csa_cp_local_pairs(const int32_t* idx, const float* scores, int32_t B, int32_t K, int64_t score_stride,
                              int64_t t0, float* pair_score, int32_t* pair_pos, csa_stream_t stream) {
  if (!idx || !scores || !pair_score || !pair_pos) return CSA_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || score_stride < 1 || t0 < 0) return CSA_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  {
    ProfScope ps(st, "cp_pairs");
    launch_k(cp_pairs_kernel, dim3(grid_for((int64_t)B * K)), dim3(256), 0, st, idx, scores, B, K, score_stride, t0,
             pair_score, pair_pos);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

size_t csa_cp_merge_workspace_size(int32_t R, int32_t B, int32_t K_local) {
  if (R < 1 || B < 1 || K_local < 1) return 0;
  const size_t n = (size_t)R * K_local;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return al((size_t)B * kHistBins * 4) + 2 * al((size_t)B * n * 4) + al((size_t)B * 4);
}

csa_status csa_cp_merge_topk(const float* pair_score, const int32_t* pair_pos, int32_t R, int32_t B,
                             int32_t K_local, int32_t K, int32_t* idx, void* workspace, size_t workspace_bytes,
                             csa_stream_t stream) {
  if (!pair_score || !pair_pos || !idx) return CSA_ERR_INVALID_ARG;
  if (R < 1 || R > 1024 || B < 1 || K_local < 1 || K < 1 || K > 65536 || (int64_t)R * K_local >= ((int64_t)1 << 31))
    return CSA_ERR_SHAPE;
  const size_t need = csa_cp_merge_workspace_size(R, B, K_local);
  if (!workspace || workspace_bytes < need) return CSA_ERR_WORKSPACE;
  if ((uintptr_t)workspace & 15) return CSA_ERR_ALIGNMENT;
  const int64_t n = (int64_t)R * K_local;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint32_t* hist = reinterpret_cast<uint32_t*>(w);
  w += al((size_t)B * kHistBins * 4);
  float* c_score = reinterpret_cast<float*>(w);
  w += al((size_t)B * n * 4);
  int32_t* c_pos = reinterpret_cast<int32_t*>(w);
  w += al((size_t)B * n * 4);
  int32_t* c_len = reinterpret_cast<int32_t*>(w);
  cudaStream_t st = (cudaStream_t)stream;
  {
    ProfScope ps(st, "cp_compact");
    launch_k(cp_compact_kernel, dim3(B), dim3(kCpThreads), 0, st, pair_score, pair_pos, R, B, K_local, c_score,
             c_pos, c_len);
  }
  note_launches(1);
  cudaError_t e = launch_zero(hist, (size_t)B * kHistBins * 4, st);
  if (e == cudaSuccess) e = launch_hist_only(c_score, n, n, c_len, hist, B, st);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  CsRow j{};
  j.vals = c_score;
  j.row_stride = n;
  j.vec = (n % 4) == 0;
  j.n = n;
  j.n_row = c_len;
  j.hist = hist;
  j.K = K;
  j.out = idx;
  j.out_stride = K;
  j.out_width = K;
  j.map = c_pos;
  j.map_stride = n;
  j.run = cs_run(n);
  return launch_cluster_select(&j, 1, B, st, "cp_merge_select") == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

csa_status csa_cp_localize(const int32_t* idx, int32_t B, int32_t K, int64_t t0, int64_t t1, int32_t* idx_local,
                           csa_stream_t stream) {
  if (!idx || !idx_local) return CSA_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || t0 < 0 || t1 < t0) return CSA_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t n = (int64_t)B * K;
  {
    ProfScope ps(st, "cp_localize");
    launch_k(cp_localize_kernel, dim3(grid_for(n)), dim3(256), 0, st, idx, n, t0, t1, idx_local);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

csa_status csa_cp_combine(const float* o_parts, const float* lse_parts, int32_t R, int32_t B, int32_t H,
                          const float* sink, float* out, float* lse, csa_stream_t stream) {
  if (!o_parts || !lse_parts || !out) return CSA_ERR_INVALID_ARG;
  if (R < 1 || R > 1024 || B < 1 || H < 1 || H > 65535) return CSA_ERR_SHAPE;
  if (((uintptr_t)o_parts & 15) || ((uintptr_t)out & 15)) return CSA_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  {
    ProfScope ps(st, "cp_combine");
    launch_k(cp_combine_kernel, dim3(B, H), dim3(128), 0, st, o_parts, lse_parts, R, B, H, sink, out, lse);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // extern "C"
