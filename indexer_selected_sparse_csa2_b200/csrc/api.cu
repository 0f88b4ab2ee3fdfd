// C ABI of the CSA2 sparse-attention step: argument checks, workspace
// layout, dispatch, and the Full / Reindex / Reuse layer stack.
//
// Layer modes follow the DeepSeek-V4.1 blog ("DeepSeek-V4.1-Flash" section,
// CSA2 paragraph: each attention layer is statically Full, Reindex or Reuse;
// main KV and indexer K are shared across layers and Top-K indices reused;
// the decoder's first Full layer builds the candidate pool later indexers
// search) and the DeepSeek-V4.1-Flash architecture database (cache-sharing
// fact: caches owned by source layers, read by the others; every layer keeps
// its own 128-token window).
#include <algorithm>
#include <atomic>
#include <mutex>

#include "select.cuh"
#include "quant.cuh"
#include "q2.cuh"

namespace csa {

static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

cudaError_t launch_quant(const void* src, int src_dtype, int64_t n_rows, int dim, int64_t src_row_stride,
                         int fmt, void* dst, int64_t dst_row_stride, cudaStream_t stream);
cudaError_t launch_quant_mx(const void* src, int src_dtype, int64_t n_rows, int dim, int64_t src_row_stride,
                            uint8_t* codes, int64_t codes_row_stride, uint8_t* scales, int64_t scales_row_stride,
                            cudaStream_t stream);
int read_mx_error(bool clear);
cudaError_t launch_compress(const void* src, int src_dtype, const float* gate, int64_t n_groups, int m, int dim,
                            int64_t src_row_stride, int64_t gate_row_stride, int fmt, void* dst,
                            int64_t dst_row_stride, cudaStream_t stream);
size_t index_decode_ws_bytes(const csa_index_args* a);
cudaError_t run_index_decode(const csa_index_args* a, void* ws, cudaStream_t stream, uint32_t* hists,
                             cudaEvent_t pool_done, int64_t safe_rows);
size_t index_hist_bytes(const csa_index_args* a);
size_t attn_ws_bytes(const csa_attn_args* a, int share);
int read_tc_error(bool clear);
int read_pf_error(bool clear);
int read_at_error(bool clear);
int read_pk_error(bool clear);
cudaError_t run_sparse_attn(const csa_attn_args* a, void* ws, cudaStream_t stream, const void* q2, int share);
bool attn_tc_path(const csa_attn_args* a);

static bool al16(const void* p) { return ((uintptr_t)p & 15) == 0; }
static bool al16i(int64_t v) { return (v & 15) == 0; }

static csa_status check_quant(const void* src, int32_t src_dtype, int64_t n_rows, int32_t dim,
                              int64_t src_row_stride, int32_t fmt, const void* dst, int64_t dst_row_stride) {
  if (src_dtype != CSA_SRC_F32 && src_dtype != CSA_SRC_BF16) return CSA_ERR_INVALID_ARG;
  if (fmt != CSA_FMT_FP4_E2M1_E4M3X16 && fmt != CSA_FMT_FP8_E4M3_UE8M0X32 && fmt != CSA_FMT_FP8_E4M3_PLAIN)
    return CSA_ERR_INVALID_ARG;
  if (n_rows < 0) return CSA_ERR_SHAPE;
  if (n_rows == 0) return CSA_OK;
  if (!src || !dst) return CSA_ERR_INVALID_ARG;
  if (fmt == CSA_FMT_FP8_E4M3_PLAIN) {
    if (dim <= 0 || dim % 16) return CSA_ERR_SHAPE;
  } else if (dim != kD) {
    return CSA_ERR_SHAPE;
  }
  const int64_t esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  if (src_row_stride < dim) return CSA_ERR_SHAPE;
  const int64_t row_bytes = fmt == CSA_FMT_FP4_E2M1_E4M3X16 ? kFp4Bytes : (fmt == CSA_FMT_FP8_E4M3_UE8M0X32 ? kFp8Bytes : dim);
  if (n_rows > 1 && dst_row_stride < row_bytes) return CSA_ERR_SHAPE;
  if (!al16(src) || !al16i(src_row_stride * esz) || !al16(dst) || !al16i(dst_row_stride)) return CSA_ERR_ALIGNMENT;
  return CSA_OK;
}

static csa_status check_index(const csa_index_args* a) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 1 || a->n_q < 1 || a->T < a->n_q || a->T >= ((int64_t)1 << 31)) return CSA_ERR_SHAPE;
  if (a->key_format == CSA_KEY_MXFP4) {
    if (a->H_I != 32 || a->d_I != 128) return CSA_ERR_SHAPE;
    if (a->n_q != 1 || a->pool) return CSA_ERR_UNSUPPORTED;
    if (!a->key_scales) return CSA_ERR_INVALID_ARG;
    if (a->key_scale_row_stride < 4 || ((uintptr_t)a->key_scales & 3) || (a->key_scale_row_stride & 3) ||
        (a->key_scale_batch_stride & 3))
      return CSA_ERR_ALIGNMENT;
    // the packed 4-bit copy into the tensor cores' operand layout
    if (((uintptr_t)a->keys & 31) || (a->key_row_stride & 31) || (a->key_batch_stride & 31)) return CSA_ERR_ALIGNMENT;
  } else if (a->key_format != CSA_KEY_E4M3) {
    return CSA_ERR_INVALID_ARG;
  } else if (a->H_I < 1 || a->H_I > 8 || a->d_I != kDI) {
    return CSA_ERR_SHAPE;
  }
  if (a->K < 1 || a->K > 65536) return CSA_ERR_SHAPE;
  if (!a->keys || !a->q || !a->w || !a->idx) return CSA_ERR_INVALID_ARG;
  if (a->key_row_stride < (a->key_format == CSA_KEY_MXFP4 ? 64 : kDI)) return CSA_ERR_SHAPE;
  if (!al16(a->keys) || !al16i(a->key_row_stride) || !al16i(a->key_batch_stride) || !al16(a->q))
    return CSA_ERR_ALIGNMENT;
  if (a->n_q > 1) {
    // prefill chunk: no pool, no score output, K within the final select's capacity
    if (a->pool || a->pool_out || a->scores) return CSA_ERR_UNSUPPORTED;
    if (a->K > 4096) return CSA_ERR_SHAPE;
    return CSA_OK;
  }
  if (a->pool && a->pool_out) return CSA_ERR_UNSUPPORTED;
  if (a->pool) {
    if (!a->pool_len || a->pool_cap < 1) return CSA_ERR_INVALID_ARG;
  }
  if (a->pool_out) {
    if (!a->pool_out_len) return CSA_ERR_INVALID_ARG;
    const int bl = a->pool_block_len;
    if (a->pool_blocks < 1 || a->pool_blocks > 65536) return CSA_ERR_SHAPE;
    if (bl != 1 && bl != 2 && bl != 4 && bl != 8 && bl != 16) return CSA_ERR_SHAPE;
  }
  return CSA_OK;
}

static csa_status check_attn(const csa_attn_args* a) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 1 || a->n_q < 1) return CSA_ERR_SHAPE;
  if (a->H != 16 && a->H != 32 && a->H != 64) return CSA_ERR_SHAPE;
  if (a->D != kD) return CSA_ERR_SHAPE;
  if (a->K < 0 || a->K > 65536 || a->n_win < 0 || a->n_win > 1024) return CSA_ERR_SHAPE;
  if (!a->q || !a->out) return CSA_ERR_INVALID_ARG;
  if (a->K > 0 && (!a->kv || !a->idx)) return CSA_ERR_INVALID_ARG;
  if (a->n_win > 0 && !a->win) return CSA_ERR_INVALID_ARG;
  if (a->K > 0 && (a->kv_row_stride < kFp4Bytes || !al16(a->kv) || !al16i(a->kv_row_stride) ||
                   !al16i(a->kv_batch_stride)))
    return a->kv_row_stride < kFp4Bytes ? CSA_ERR_SHAPE : CSA_ERR_ALIGNMENT;
  if (a->n_win > 0 && (a->win_row_stride < kFp8Bytes || !al16(a->win) || !al16i(a->win_row_stride) ||
                       !al16i(a->win_batch_stride)))
    return a->win_row_stride < kFp8Bytes ? CSA_ERR_SHAPE : CSA_ERR_ALIGNMENT;
  if (!al16(a->q) || !al16(a->out) || !al16(a->rope_cs)) return CSA_ERR_ALIGNMENT;
  if (a->out_bf16 != 0 && a->out_bf16 != 1) return CSA_ERR_INVALID_ARG;
  return CSA_OK;
}

static csa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

}  // namespace csa

using namespace csa;

extern "C" {

csa_status csa_quant_kv(const void* src, int32_t src_dtype, int64_t n_rows, int32_t dim,
                        int64_t src_row_stride, int32_t fmt, void* dst, int64_t dst_row_stride,
                        csa_stream_t stream) {
  csa_status s = check_quant(src, src_dtype, n_rows, dim, src_row_stride, fmt, dst, dst_row_stride);
  if (s != CSA_OK || n_rows == 0) return s;
  return from_cuda(launch_quant(src, src_dtype, n_rows, dim, src_row_stride, fmt, dst, dst_row_stride,
                                (cudaStream_t)stream));
}

csa_status csa_compress_kv(const void* src, int32_t src_dtype, const float* gate, int64_t n_groups, int32_t m,
                           int32_t dim, int64_t src_row_stride, int64_t gate_row_stride, int32_t fmt, void* dst,
                           int64_t dst_row_stride, csa_stream_t stream) {
  if (src_dtype != CSA_SRC_F32 && src_dtype != CSA_SRC_BF16) return CSA_ERR_INVALID_ARG;
  if (fmt != CSA_FMT_FP4_E2M1_E4M3X16 && fmt != CSA_FMT_FP8_E4M3_PLAIN) return CSA_ERR_INVALID_ARG;
  if (n_groups < 0 || m < 1 || m > 16) return CSA_ERR_SHAPE;
  if (n_groups == 0) return CSA_OK;
  if (!src || !dst || (m > 1 && !gate)) return CSA_ERR_INVALID_ARG;
  if (fmt == CSA_FMT_FP4_E2M1_E4M3X16 ? dim != kD : (dim <= 0 || dim % 16)) return CSA_ERR_SHAPE;
  if (src_row_stride < dim || (m > 1 && gate_row_stride < dim)) return CSA_ERR_SHAPE;
  const int64_t esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  const int64_t row_bytes = fmt == CSA_FMT_FP4_E2M1_E4M3X16 ? kFp4Bytes : dim;
  if (n_groups > 1 && dst_row_stride < row_bytes) return CSA_ERR_SHAPE;
  if (!al16(src) || !al16i(src_row_stride * esz) || !al16(dst) || !al16i(dst_row_stride)) return CSA_ERR_ALIGNMENT;
  if (m > 1 && (!al16(gate) || !al16i(gate_row_stride * 4))) return CSA_ERR_ALIGNMENT;
  return from_cuda(launch_compress(src, src_dtype, gate, n_groups, m, dim, src_row_stride, gate_row_stride, fmt, dst,
                                   dst_row_stride, (cudaStream_t)stream));
}

csa_status csa_quant_mxfp4(const void* src, int32_t src_dtype, int64_t n_rows, int32_t dim, int64_t src_row_stride,
                           uint8_t* codes, int64_t codes_row_stride, uint8_t* scales, int64_t scales_row_stride,
                           csa_stream_t stream) {
  if (src_dtype != CSA_SRC_F32 && src_dtype != CSA_SRC_BF16) return CSA_ERR_INVALID_ARG;
  if (n_rows < 0 || dim <= 0 || dim % 32) return CSA_ERR_SHAPE;
  if (n_rows == 0) return CSA_OK;
  if (!src || !codes || !scales) return CSA_ERR_INVALID_ARG;
  if (src_row_stride < dim || (n_rows > 1 && (codes_row_stride < dim / 2 || scales_row_stride < dim / 32)))
    return CSA_ERR_SHAPE;
  const int64_t esz = src_dtype == CSA_SRC_BF16 ? 2 : 4;
  if (!al16(src) || !al16i(src_row_stride * esz) || !al16(codes) || !al16i(codes_row_stride)) return CSA_ERR_ALIGNMENT;
  return from_cuda(launch_quant_mx(src, src_dtype, n_rows, dim, src_row_stride, codes, codes_row_stride, scales,
                                   scales_row_stride, (cudaStream_t)stream));
}

size_t csa_index_workspace_size(const csa_index_args* a) {
  if (check_index(a) != CSA_OK) return 0;
  return index_decode_ws_bytes(a);
}

csa_status csa_index_topk(const csa_index_args* a, void* workspace, size_t workspace_bytes,
                          csa_stream_t stream) {
  csa_status s = check_index(a);
  if (s != CSA_OK) return s;
  const size_t need = index_decode_ws_bytes(a);
  if (need > workspace_bytes || (need && !workspace)) return CSA_ERR_WORKSPACE;
  if (!al16(workspace)) return CSA_ERR_ALIGNMENT;
  return from_cuda(run_index_decode(a, workspace, (cudaStream_t)stream, nullptr, nullptr, -1));
}

size_t csa_topk_workspace_size(int32_t B, int64_t n) {
  if (B < 1 || n < 1) return 0;
  return ((size_t)B * kHistBins * 4 + 255) & ~(size_t)255;
}

csa_status csa_topk_scores(const float* scores, int32_t B, int64_t n, int64_t row_stride, int32_t K,
                           int32_t* idx, void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  if (!scores || !idx) return CSA_ERR_INVALID_ARG;
  if (B < 1 || n < 1 || n >= ((int64_t)1 << 31) || row_stride < n || K < 1 || K > 65536) return CSA_ERR_SHAPE;
  const size_t need = csa_topk_workspace_size(B, n);
  if (need > workspace_bytes || !workspace) return CSA_ERR_WORKSPACE;
  if (!al16(workspace)) return CSA_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* hist = static_cast<uint32_t*>(workspace);
  cudaError_t e = launch_zero(hist, (size_t)B * kHistBins * 4, st);
  if (e == cudaSuccess) e = launch_hist_only(scores, row_stride, n, nullptr, hist, B, st);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  CsRow j{};
  j.vals = scores;
  j.row_stride = row_stride;
  j.vec = (row_stride % 4) == 0 && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  j.n = n;
  j.hist = hist;
  j.K = K;
  j.out = idx;
  j.out_stride = K;
  j.out_width = K;
  j.run = cs_run(n);
  return from_cuda(launch_cluster_select(&j, 1, B, st, "topk_select"));
}

size_t csa_attn_workspace_size(const csa_attn_args* a) {
  if (check_attn(a) != CSA_OK) return 0;
  return attn_ws_bytes(a, 1);
}

csa_status csa_sparse_attn(const csa_attn_args* a, void* workspace, size_t workspace_bytes,
                           csa_stream_t stream) {
  csa_status s = check_attn(a);
  if (s != CSA_OK) return s;
  const size_t need = attn_ws_bytes(a, 1);
  if (need > workspace_bytes || (need && !workspace)) return CSA_ERR_WORKSPACE;
  if (need && !al16(workspace)) return CSA_ERR_ALIGNMENT;
  return from_cuda(run_sparse_attn(a, workspace, (cudaStream_t)stream, nullptr, 1));
}

// Layers that run the indexer (Full, Reindex); Reuse and SWA layers do not.
static bool indexes(int32_t mode) { return mode == CSA_MODE_FULL || mode == CSA_MODE_REINDEX; }

// Resolve one layer of a stack into concrete index / attention arguments.
static csa_status resolve_layer(const csa_layer_desc* L, int32_t i, csa_index_args* ix, csa_attn_args* at) {
  const csa_layer_desc& d = L[i];
  *at = d.attn;
  if (d.mode == CSA_MODE_SWA) {
    at->idx = nullptr;
    at->K = 0;
    return CSA_OK;
  }
  if (d.mode == CSA_MODE_REUSE) {
    if (d.reuse_from < 0 || d.reuse_from >= i) return CSA_ERR_INVALID_ARG;
    int32_t src = d.reuse_from;
    while (L[src].mode == CSA_MODE_REUSE) {            // a chain of reuse resolves to its source
      if (L[src].reuse_from < 0 || L[src].reuse_from >= src) return CSA_ERR_INVALID_ARG;
      src = L[src].reuse_from;
    }
    if (L[src].mode == CSA_MODE_SWA) return CSA_ERR_INVALID_ARG;   // a window layer has no indices
    if (L[src].index.n_q != at->n_q || L[src].index.B != at->B) return CSA_ERR_SHAPE;
    at->idx = L[src].index.idx;
    at->K = L[src].index.K;
    return CSA_OK;
  }
  if (d.mode != CSA_MODE_FULL && d.mode != CSA_MODE_REINDEX) return CSA_ERR_INVALID_ARG;
  *ix = d.index;
  if (d.mode == CSA_MODE_REINDEX && d.pool_from >= 0) {
    if (d.pool_from >= i || !L[d.pool_from].index.pool_out) return CSA_ERR_INVALID_ARG;
    const csa_index_args& P = L[d.pool_from].index;
    ix->pool = P.pool_out;
    ix->pool_len = P.pool_out_len;
    ix->pool_cap = P.pool_blocks * P.pool_block_len;
    ix->pool_out = nullptr;
    ix->pool_out_len = nullptr;
  } else if (d.mode == CSA_MODE_REINDEX) {
    ix->pool = nullptr;
  }
  if (d.mode == CSA_MODE_FULL) ix->pool = nullptr;
  if (ix->n_q != at->n_q || ix->B != at->B) return CSA_ERR_SHAPE;
  at->idx = ix->idx;
  at->K = ix->K;
  return CSA_OK;
}

// Workspace of a layer stack: one region per layer (a layer's index scratch
// and its attention partials; layers may run concurrently, so regions are not
// shared), then one histogram region per indexed decode layer (all cleared by
// the prologue launch), then the staged decode queries.
struct StackWs {
  size_t layers = 0;       // total of the per-layer regions
  size_t hists = 0;        // total of the per-layer histogram regions
  size_t q2 = 0;           // total of the per-layer staged decode queries
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

// Decode layers on the tcgen05 attention kernel get their queries staged by
// the prologue (one copy per token instead of a conversion per split CTA).
static size_t layer_q2_bytes(const csa_attn_args& at) {
  if (at.n_q != 1 || !attn_tc_path(&at)) return 0;
  return al256((size_t)at.B * kQ2TokenBytes);
}

// Source layer of a Reuse chain.
static int32_t reuse_source(const csa_layer_desc* L, int32_t i) {
  int32_t src = L[i].reuse_from;
  while (L[src].mode == CSA_MODE_REUSE) src = L[src].reuse_from;
  return src;
}

// Dependency wave of a layer of a validated stack: 0 for layers that wait only
// for the prologue (Full, Reindex over all positions), otherwise one more than
// the wave of the layer whose pool (Reindex in a pool) or Top-K (Reuse) it
// waits for.  Layers of one wave run their attention at about the same time,
// so each plans its split grid for its share of the SMs.
static int layer_wave(const csa_layer_desc* L, int32_t i) {
  if (L[i].mode == CSA_MODE_REUSE) return 1 + layer_wave(L, reuse_source(L, i));
  if (L[i].mode == CSA_MODE_REINDEX && L[i].pool_from >= 0) return 1 + layer_wave(L, L[i].pool_from);
  return 0;
}

static int attn_share(const csa_layer_desc* L, int32_t n_layers, int32_t i) {
  const int w = layer_wave(L, i);
  int c = 0;
  for (int32_t j = 0; j < n_layers; ++j) c += layer_wave(L, j) == w;
  return c;
}

static size_t layer_region_bytes(const csa_layer_desc& L, const csa_index_args& ix, const csa_attn_args& at,
                                 int share) {
  size_t r = attn_ws_bytes(&at, share);
  if (indexes(L.mode)) r = std::max(r, index_decode_ws_bytes(&ix));
  return al256(r);
}

// The first key row of `ix` that the stack's prologue (every layer's append
// jobs) writes, for the full scan that overlaps the prologue: rows below it may
// be read before the prologue ends.  -1 (wait first) when a job writes the
// query or the head weights.  MXFP4 keys are read only after the wait (0: no
// row early, the query and weights may be).
static int64_t prologue_safe_rows(const csa_layer_desc* layers, int32_t n_layers, const csa_index_args& ix) {
  const bool mx = ix.key_format == CSA_KEY_MXFP4;
  if ((ix.key_format != CSA_KEY_E4M3 && !mx) || ix.pool || ix.n_q != 1 || ix.T <= 0) return -1;
  const int64_t bs = ix.key_batch_stride ? ix.key_batch_stride : ix.key_row_stride * ix.T;
  const uintptr_t k0 = reinterpret_cast<uintptr_t>(ix.keys);
  const uintptr_t k1 = k0 + (uintptr_t)((ix.B - 1) * bs + ix.T * ix.key_row_stride);
  const uintptr_t q0 = reinterpret_cast<uintptr_t>(ix.q), q1 = q0 + (uintptr_t)ix.B * ix.H_I * ix.d_I;
  const uintptr_t w0 = reinterpret_cast<uintptr_t>(ix.w), w1 = w0 + (uintptr_t)ix.B * ix.H_I * 4;
  int64_t safe = mx ? 0 : ix.T;
  for (int32_t i = 0; i < n_layers; ++i) {
    for (int k = 0; k < 3; ++k) {
      const csa_quant_job& q = layers[i].append[k];
      if (!q.src || q.n_rows <= 0) continue;
      const int64_t rb = q.fmt == CSA_FMT_FP4_E2M1_E4M3X16 ? kFp4Bytes
                         : (q.fmt == CSA_FMT_FP8_E4M3_UE8M0X32 ? kFp8Bytes : q.dim);
      for (int64_t j = 0; j < q.n_rows; ++j) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(q.dst) + (uintptr_t)(j * q.dst_row_stride);
        const uintptr_t a1 = a0 + (uintptr_t)rb;
        if (a0 < q1 && a1 > q0) return -1;
        if (a0 < w1 && a1 > w0) return -1;
        if (mx || a0 >= k1 || a1 <= k0) continue;
        // the rows this write touches (from its first and last byte)
        for (uintptr_t a : {a0 < k0 ? k0 : a0, (a1 > k1 ? k1 : a1) - 1}) {
          const int64_t off = (int64_t)(a - k0);
          const int64_t t = (off % bs) / ix.key_row_stride;
          if (t < safe) safe = t;
        }
        if (a1 - a0 > (uintptr_t)ix.key_row_stride) safe = 0;   // spans rows: be safe
      }
    }
  }
  return safe;
}

static csa_status stack_ws(const csa_layer_desc* layers, int32_t n_layers, StackWs* out) {
  StackWs w;
  for (int32_t i = 0; i < n_layers; ++i) {
    csa_index_args ix{};
    csa_attn_args at{};
    csa_status s = resolve_layer(layers, i, &ix, &at);
    if (s != CSA_OK) return s;
    for (int k = 0; k < 3; ++k) {
      const csa_quant_job& q = layers[i].append[k];
      if (!q.src) continue;
      s = check_quant(q.src, q.src_dtype, q.n_rows, q.dim, q.src_row_stride, q.fmt, q.dst, q.dst_row_stride);
      if (s != CSA_OK) return s;
    }
    if (indexes(layers[i].mode)) {
      s = check_index(&ix);
      if (s != CSA_OK) return s;
      w.hists += index_hist_bytes(&ix);
    }
    s = check_attn(&at);
    if (s != CSA_OK) return s;
    w.q2 += layer_q2_bytes(at);
  }
  // every layer is valid: the waves (and the split grids they set) are defined
  for (int32_t i = 0; i < n_layers; ++i) {
    csa_index_args ix{};
    csa_attn_args at{};
    resolve_layer(layers, i, &ix, &at);
    w.layers += layer_region_bytes(layers[i], ix, at, attn_share(layers, n_layers, i));
  }
  *out = w;
  return CSA_OK;
}

size_t csa_layer_workspace_size(const csa_layer_desc* layers, int32_t n_layers) {
  if (!layers || n_layers < 1) return 0;
  StackWs w;
  if (stack_ws(layers, n_layers, &w) != CSA_OK) return 0;
  return w.layers + w.hists + w.q2;
}

// Host-side streams and events the stack uses to run independent layers
// concurrently (created once per device; no device memory).  Under stream
// capture the fork / join below becomes graph edges.
// Auxiliary streams per device: the last stages the decode queries, the
// others carry layers 1, 2, ... in turn.  Enough that the independent chains
// of a deep stack (a 40-layer stack has 4 Full layers and their Reuse layers)
// rarely queue behind one another on a shared stream.
constexpr int kAuxStreams = 32;
constexpr int kLayerStreams = kAuxStreams - 1;
constexpr int kMaxStackLayers = 64;
static_assert(sizeof(csa_step_sync::layer_done) / sizeof(void*) == kMaxStackLayers, "csa_step_sync layout");
struct StackStreams {
  cudaStream_t aux[kAuxStreams] = {};
  cudaEvent_t start = nullptr;   // the caller's stream at the start of a step
  cudaEvent_t pro = nullptr;     // prologue (appends, histogram clearing) done
  cudaEvent_t stg = nullptr;     // decode queries staged
  cudaEvent_t idx[kMaxStackLayers] = {};
  cudaEvent_t pool[kMaxStackLayers] = {};   // a pool-building layer's pool is written
  cudaEvent_t join[kAuxStreams] = {};   // tail of an auxiliary stream, joined into the caller's
  std::mutex mu;                        // one step enqueues on this device's streams at a time
  bool ok = false;
};
static std::mutex g_stack_mu;
static StackStreams g_stack[64];

static StackStreams* stack_streams() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_stack_mu);
  StackStreams& S = g_stack[dev];
  if (!S.ok) {
    bool good = true;
    for (int i = 0; i < kAuxStreams && good; ++i)
      good = cudaStreamCreateWithFlags(&S.aux[i], cudaStreamNonBlocking) == cudaSuccess;
    good = good && cudaEventCreateWithFlags(&S.pro, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&S.start, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&S.stg, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kMaxStackLayers && good; ++i)
      good = cudaEventCreateWithFlags(&S.idx[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&S.pool[i], cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kAuxStreams && good; ++i)
      good = cudaEventCreateWithFlags(&S.join[i], cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    S.ok = true;
  }
  return &S;
}

csa_status csa_layer_step(const csa_layer_desc* layers, int32_t n_layers, void* workspace,
                          size_t workspace_bytes, csa_stream_t stream) {
  return csa_layer_step_sync(layers, n_layers, workspace, workspace_bytes, nullptr, stream);
}

csa_status csa_layer_step_sync(const csa_layer_desc* layers, int32_t n_layers, void* workspace,
                               size_t workspace_bytes, const csa_step_sync* sync, csa_stream_t stream) {
  if (!layers || n_layers < 1) return CSA_ERR_INVALID_ARG;
  if (n_layers > kMaxStackLayers) return CSA_ERR_UNSUPPORTED;
  // validate everything before enqueuing anything
  StackWs w;
  csa_status s = stack_ws(layers, n_layers, &w);
  if (s != CSA_OK) return s;
  const size_t need = w.layers + w.hists + w.q2;
  if (need > workspace_bytes || (need && !workspace)) return CSA_ERR_WORKSPACE;
  if (need && !al16(workspace)) return CSA_ERR_ALIGNMENT;
  StackStreams* SS = stack_streams();
  if (!SS) return CSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // The step enqueues on library-owned auxiliary streams and events of this
  // device: one caller at a time, and every auxiliary stream it used is
  // joined into the caller's stream again, also when a launch fails half way.
  std::lock_guard<std::mutex> lk(SS->mu);
  bool used[kAuxStreams] = {};
  auto enqueue = [&]() -> csa_status {
    uint8_t* base = static_cast<uint8_t*>(workspace);
    uint8_t* hist_base = base + w.layers;
    uint8_t* q2_base = hist_base + w.hists;

    // prologue on the caller's stream: every layer's appended rows and the
    // clearing of every layer's histograms, in one launch (each layer reads only
    // rows appended before it in stream order, so moving the appends ahead of
    // all layers is the same).  The staging of the decode queries, which only
    // the attention kernels read, runs on an auxiliary stream beside the first
    // layer's scoring.
    QuantBatch qb{}, qs{};
    qb.zero_ptr = reinterpret_cast<uint4*>(hist_base);
    qb.zero_n16 = (int64_t)(w.hists / 16);
    cudaStream_t sst = SS->aux[kAuxStreams - 1];
    auto add_job = [&](QuantBatch& q, cudaStream_t qs_stream, const void* src, int64_t n_rows,
                       int64_t src_stride_bytes, void* dst, int64_t dst_stride, int fmt, int bf16, int dim,
                       const float* aux) -> bool {
      if (q.njobs == kMaxBatchJobs) {
        if (launch_quant_batch(q, qs_stream) != cudaSuccess) return false;
        q.njobs = 0;
        q.units = 0;
        q.zero_n16 = 0;
      }
      QuantBatchJob& J = q.job[q.njobs++];
      J.src = src;
      J.n_rows = n_rows;
      J.src_stride_bytes = src_stride_bytes;
      J.dst = static_cast<uint8_t*>(dst);
      J.dst_stride = dst_stride;
      J.fmt = fmt;
      J.bf16 = bf16;
      J.dim = dim;
      J.aux = aux;
      J.unit0 = q.units;
      q.units += quant_batch_units(fmt, n_rows, dim);
      return true;
    };
    const bool staged = w.q2 > 0;
    cudaEvent_t q_ready = sync ? static_cast<cudaEvent_t>(sync->queries_ready) : nullptr;
    if (staged) {
      used[kAuxStreams - 1] = true;
      if (cudaEventRecord(SS->start, st) != cudaSuccess || cudaStreamWaitEvent(sst, SS->start, 0) != cudaSuccess)
        return CSA_ERR_CUDA;
      // the staging is the first reader of the attention queries
      if (q_ready && cudaStreamWaitEvent(sst, q_ready, 0) != cudaSuccess) return CSA_ERR_CUDA;
    }
    size_t q2_off = 0;
    for (int32_t i = 0; i < n_layers; ++i) {
      for (int k = 0; k < 3; ++k) {
        const csa_quant_job& q = layers[i].append[k];
        if (!q.src || q.n_rows == 0) continue;
        const int esz = q.src_dtype == CSA_SRC_BF16 ? 2 : 4;
        if (!add_job(qb, st, q.src, q.n_rows, q.src_row_stride * esz, q.dst, q.dst_row_stride, q.fmt,
                     q.src_dtype == CSA_SRC_BF16, q.dim, nullptr))
          return CSA_ERR_CUDA;
      }
      csa_index_args ix{};
      csa_attn_args at{};
      resolve_layer(layers, i, &ix, &at);
      if (layer_q2_bytes(at)) {
        if (!add_job(qs, sst, at.q, (int64_t)at.B * 64, 0, q2_base + q2_off, kQ2TokenBytes, kFmtStageQ2, 0, 512,
                     at.rope_cs))
          return CSA_ERR_CUDA;
        q2_off += layer_q2_bytes(at);
      }
    }
    if (launch_quant_batch(qb, st) != cudaSuccess) return CSA_ERR_CUDA;
    if (cudaEventRecord(SS->pro, st) != cudaSuccess) return CSA_ERR_CUDA;
    if (staged) {
      if (launch_quant_batch(qs, sst) != cudaSuccess) return CSA_ERR_CUDA;
      if (cudaEventRecord(SS->stg, sst) != cudaSuccess) return CSA_ERR_CUDA;
    }

    // Layers run concurrently where the mode stack allows it: layer 0 on the
    // caller's stream, layer i > 0 on an auxiliary stream that waits for the
    // prologue, for the pool builder's Top-K (Reindex in a pool) or for the
    // reused layer's Top-K (Reuse); the caller's stream then waits for all.
    size_t reg_off = 0, hist_off = 0;
    q2_off = 0;
    for (int32_t i = 0; i < n_layers; ++i) {
      csa_index_args ix{};
      csa_attn_args at{};
      resolve_layer(layers, i, &ix, &at);
      const csa_layer_desc& L = layers[i];
      if (i > 0) used[(i - 1) % kLayerStreams] = true;
      cudaStream_t ls = i == 0 ? st : SS->aux[(i - 1) % kLayerStreams];
      if (i > 0 && cudaStreamWaitEvent(ls, SS->pro, 0) != cudaSuccess) return CSA_ERR_CUDA;
      uint8_t* region = base + reg_off;
      const int share = attn_share(layers, n_layers, i);
      reg_off += layer_region_bytes(L, ix, at, share);
      if (indexes(L.mode)) {
        if (L.mode == CSA_MODE_REINDEX && L.pool_from >= 0 && cudaStreamWaitEvent(ls, SS->pool[L.pool_from], 0) != cudaSuccess)
          return CSA_ERR_CUDA;
        uint32_t* h = index_hist_bytes(&ix) ? reinterpret_cast<uint32_t*>(hist_base + hist_off) : nullptr;
        hist_off += index_hist_bytes(&ix);
        if (run_index_decode(&ix, region, ls, h, ix.pool_out ? SS->pool[i] : nullptr,
                             prologue_safe_rows(layers, n_layers, ix)) != cudaSuccess)
          return CSA_ERR_CUDA;
      } else if (L.mode == CSA_MODE_REUSE &&
                 cudaStreamWaitEvent(ls, SS->idx[reuse_source(layers, i)], 0) != cudaSuccess) {
        return CSA_ERR_CUDA;
      }
      if (cudaEventRecord(SS->idx[i], ls) != cudaSuccess) return CSA_ERR_CUDA;
      const void* q2 = layer_q2_bytes(at) ? q2_base + q2_off : nullptr;
      q2_off += layer_q2_bytes(at);
      if (q2 && cudaStreamWaitEvent(ls, SS->stg, 0) != cudaSuccess) return CSA_ERR_CUDA;
      if (!q2 && q_ready && cudaStreamWaitEvent(ls, q_ready, 0) != cudaSuccess) return CSA_ERR_CUDA;
      if (run_sparse_attn(&at, region, ls, q2, share) != cudaSuccess) return CSA_ERR_CUDA;
      if (sync && sync->layer_done[i] && cudaEventRecord(static_cast<cudaEvent_t>(sync->layer_done[i]), ls) != cudaSuccess)
        return CSA_ERR_CUDA;
    }
    return CSA_OK;
  };
  const csa_status rc = enqueue();
  for (int k = 0; k < kAuxStreams; ++k) {
    if (!used[k]) continue;
    if (cudaEventRecord(SS->join[k], SS->aux[k]) != cudaSuccess || cudaStreamWaitEvent(st, SS->join[k], 0) != cudaSuccess)
      return CSA_ERR_CUDA;
  }
  return rc;
}

const char* csa_status_string(int32_t s) {
  switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_SHAPE: return "unsupported or inconsistent shape";
    case CSA_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case CSA_ERR_UNSUPPORTED: return "unsupported combination";
    case CSA_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
  }
}

int32_t csa_device_status(void) {
  const int a = read_tc_error(true), b = read_pf_error(true), c = read_at_error(true);
  const int d = read_pk_error(true), e = read_mx_error(true);
  return (int32_t)(a ? a : (b ? b : (c ? c : (d ? d : e))));
}

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }
int32_t csa_version(void) { return 1; }

}  // extern "C"
