/*
 * csa.h - C ABI of the CSA2 compressed sparse-attention step (sm_100a).
 *
 * The step, per decode (or prefill) token of one attention layer:
 *   (a) encode main-KV latents as FP4 E2M1 with one E4M3 scale per 16
 *       channels (288-byte entries), the sliding-window KV as FP8 E4M3 with
 *       one UE8M0 scale per 32 channels (528-byte entries), and indexer keys /
 *       queries as plain E4M3;
 *   (b) score every cached position (or a candidate pool) with the lightning
 *       indexer S[s] = sum_j w[j] * relu(<qI[j], kI[s]>) and keep the Top-K;
 *   (c) MLA attention of the query heads over the selected FP4 entries plus
 *       the FP8 window (keys = values = the 512-wide dequantised latent).
 * Layers run in one of three modes: Full, Reindex, Reuse.
 *
 * Sources: DeepSeek-V4.1 blog, "DeepSeek-V4.1-Flash" section, CSA2 paragraph
 * (modes, hierarchical indexer, FP4 main KV with E4M3 per 16 channels);
 * DeepSeek-V4.1-Flash architecture database (cache owners and sharing, entry
 * storage formats, "2048-block x 8-position candidate pool");
 * Model techniques map - DeepSeek-V4.1-Flash ("Indexer-selected sparse
 * attention", "Sliding-window attention", "Learnable attention sink",
 * "Multi-head latent attention" rows).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates, frees or synchronises; work is enqueued on
 *     `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Transient memory is the caller's `workspace`, sized by the matching
 *     *_workspace_size() call (0 bytes is valid when the size is 0).
 *   - Arguments are checked on the host before any launch; a failed check
 *     returns a non-zero csa_status and enqueues nothing.  A failed launch
 *     returns CSA_ERR_CUDA.
 *   - Byte strides and entry pointers must be 16-byte aligned.
 *   - Calls keep no device state between them and may be captured in a
 *     CUDA graph (csa_layer_step keeps host-side streams and events per
 *     device; see there).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t;

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1, /* NULL where a pointer is required, unknown enum */
  CSA_ERR_SHAPE = 2,       /* a size outside the supported range */
  CSA_ERR_ALIGNMENT = 3,   /* pointer or stride not 16-byte aligned */
  CSA_ERR_UNSUPPORTED = 4, /* valid combination that is not implemented */
  CSA_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than required */
  CSA_ERR_CUDA = 6         /* a kernel launch failed */
} csa_status;

typedef enum { CSA_SRC_F32 = 0, CSA_SRC_BF16 = 1 } csa_src_dtype;

typedef enum {
  /* 512 channels -> 288 B: bytes 0..255 = E2M1 codes, two per byte, even
   * channel in the low nibble; bytes 256..287 = E4M3 scale of each block of
   * 16 channels.  scale = E4M3_rne_sat(amax/6); code = E2M1_rne_sat(x/scale)
   * (fp32 IEEE divisions); a zero scale gives all codes +0. */
  CSA_FMT_FP4_E2M1_E4M3X16 = 0,
  /* 512 channels -> 528 B: bytes 0..511 = E4M3 codes; bytes 512..527 = UE8M0
   * exponent byte (e + 127) of each block of 32 channels, where e is the
   * smallest integer with amax <= 448 * 2^e, clamped to [-127, 127];
   * code = E4M3_rne_sat(x * 2^-e). */
  CSA_FMT_FP8_E4M3_UE8M0X32 = 1,
  /* dim channels -> dim bytes of E4M3_rne_sat(x) (indexer keys/queries). */
  CSA_FMT_FP8_E4M3_PLAIN = 2
} csa_kv_format;

/* SWA: a sliding-window layer (the stack's first layers): attention over the
 * layer's window alone, no indexer, no selected entries. */
typedef enum { CSA_MODE_FULL = 0, CSA_MODE_REINDEX = 1, CSA_MODE_REUSE = 2, CSA_MODE_SWA = 3 } csa_mode;

/* ------------------------------------------------------------------------ */
/* (a) Encode rows.
 *   src            : n_rows rows of `dim` fp32 or bf16 values, row r at
 *                    src + r * src_row_stride elements.
 *   dim            : 512 for the FP4 / windowed FP8 formats; a positive
 *                    multiple of 16 for CSA_FMT_FP8_E4M3_PLAIN.
 *   dst            : row r written at dst + r * dst_row_stride bytes
 *                    (288, 528 or dim bytes per row).
 * Encodings are bit-exact functions of the inputs (round to nearest even,
 * saturating); see csa_kv_format.  Non-finite inputs are outside the
 * contract. */
csa_status csa_quant_kv(const void* src, int32_t src_dtype, int64_t n_rows, int32_t dim,
                        int64_t src_row_stride, int32_t fmt, void* dst,
                        int64_t dst_row_stride, csa_stream_t stream);

/* The m-token compressor of the encoder's CSA2 layers (DeepSeek-V4.1-Flash
 * architecture database, cache groups: the encoder's main KV and indexer K
 * hold one shared K=V entry per 2 tokens, pooled with a gate in fp32; the
 * ratio-1 compressor is plain).  Group n pools token rows n*m .. n*m+m-1:
 * per channel, w_i = exp(g_i - max_j g_j) and entry = sum_i w_i x_i /
 * sum_i w_i (fp32, exp and a correctly rounded division), then the entry is
 * encoded as fmt (CSA_FMT_FP4_E2M1_E4M3X16 with dim 512, or
 * CSA_FMT_FP8_E4M3_PLAIN with dim a multiple of 16).
 *   src  : fp32 / bf16 token rows, row r at src + r * src_row_stride elements
 *   gate : fp32 gate logits, row r at gate + r * gate_row_stride (NULL when m == 1)
 *   dst  : entry n at dst + n * dst_row_stride bytes; 1 <= m <= 16.
 * Entries of an incomplete tail group are the caller's to withhold. */
csa_status csa_compress_kv(const void* src, int32_t src_dtype, const float* gate, int64_t n_groups, int32_t m,
                           int32_t dim, int64_t src_row_stride, int64_t gate_row_stride, int32_t fmt, void* dst,
                           int64_t dst_row_stride, csa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* (b) Lightning-indexer scores + Top-K (optionally building or searching the
 * hierarchical candidate pool).
 *
 * Query t (0 <= t < n_q) of sequence b sits at position T - n_q + t and
 * scores positions [0, T - n_q + t]  (decode: n_q = 1, all of [0, T)).
 *   S[s] = sum_j w[b,t,j] * max(0, sum_d qI[b,t,j,d] * kI[b,s,d])
 * Top-K keeps the K largest S, ties broken towards the lower position, and
 * writes the positions ASCENDING to idx[b,t,0..K), padding with -1 when fewer
 * than K candidates exist.
 *
 * Pool search (pool != NULL, decode only): the candidates of sequence b are
 * the positions pool[b, 0..pool_len[b]) (ascending, as written by pool_out).
 * Pool build (pool_out != NULL, decode only): positions are grouped in
 * aligned blocks of pool_block_len; a block scores the max of its positions;
 * the pool_blocks best blocks (ties -> lower block) give pool_out[b] =
 * their positions ascending (-1 padded to pool_blocks*pool_block_len) and
 * pool_out_len[b] = the number of valid positions.
 */
typedef struct {
  int32_t B;                 /* sequences, >= 1 */
  int32_t n_q;               /* query tokens per sequence, >= 1 */
  int64_t T;                 /* cache length, n_q <= T < 2^31 */
  int32_t H_I;               /* indexer heads, 1..8 */
  int32_t d_I;               /* indexer head dim; must be 64 */
  const uint8_t* keys;       /* E4M3 key of position s of sequence b at
                                keys + b*key_batch_stride + s*key_row_stride */
  int64_t key_row_stride;    /* bytes, >= 64, multiple of 16 */
  int64_t key_batch_stride;  /* bytes, multiple of 16 */
  const uint8_t* q;          /* E4M3 [B][n_q][H_I][64], contiguous */
  const float* w;            /* fp32 [B][n_q][H_I], contiguous */
  int32_t K;                 /* 1..65536 (1..4096 when n_q > 1) */
  const int32_t* pool;       /* optional [B][pool_cap] ascending positions */
  const int32_t* pool_len;   /* [B] valid entries of pool (required with pool) */
  int32_t pool_cap;          /* row length of pool */
  int32_t* pool_out;         /* optional [B][pool_blocks*pool_block_len] */
  int32_t* pool_out_len;     /* [B] (required with pool_out) */
  int32_t pool_blocks;       /* blocks kept in the pool, 1..65536 */
  int32_t pool_block_len;    /* positions per block: 1, 2, 4, 8 or 16 */
  int32_t* idx;              /* out: int32 [B][n_q][K] */
  float* scores;             /* optional out (decode only): fp32 scores
                                [B][T] (or [B][pool_cap] when searching a
                                pool; slots past pool_len are not written) */
  /* Indexer-key format.  CSA_KEY_E4M3: plain E4M3 keys (d_I = 64, H_I <= 8,
   * the fields below unused).  CSA_KEY_MXFP4: the pages' MXFP4 keys
   * (architecture database, indexer K: E2M1 with one E8M0 scale per 32
   * channels; techniques map: 32 heads x 128): d_I = 128, H_I = 32, decode
   * scans only (no pool search); `keys` holds the E2M1 codes (64 bytes per
   * key, even channel in the low nibble; `keys` 32-byte aligned and both key
   * strides multiples of 32, else CSA_ERR_ALIGNMENT) and `key_scales` the 4 exponent
   * bytes (e + 127, block order) of key s at key_scales +
   * b*key_scale_batch_stride + s*key_scale_row_stride (strides multiples of
   * 4).  Block b of the key contributes 2^e_b * <q block b, E2M1 codes>. */
  int32_t key_format;
  const uint8_t* key_scales;
  int64_t key_scale_row_stride;
  int64_t key_scale_batch_stride;
} csa_index_args;

typedef enum { CSA_KEY_E4M3 = 0, CSA_KEY_MXFP4 = 1 } csa_key_format;

/* MXFP4 encoding of indexer keys into the two planes above: per block of 32
 * channels, e = the smallest integer with amax <= 6 * 2^e, clamped to
 * [-127, 127] (amax = 0 -> -127); codes E2M1_rne_sat(x * 2^-e).
 * src: n_rows rows of `dim` (a multiple of 32) fp32 / bf16 values, row r at
 * src + r * src_row_stride elements; codes row r at codes + r *
 * codes_row_stride (dim / 2 bytes), exponent bytes at scales + r *
 * scales_row_stride (dim / 32 bytes). */
csa_status csa_quant_mxfp4(const void* src, int32_t src_dtype, int64_t n_rows, int32_t dim, int64_t src_row_stride,
                           uint8_t* codes, int64_t codes_row_stride, uint8_t* scales, int64_t scales_row_stride,
                           csa_stream_t stream);

size_t csa_index_workspace_size(const csa_index_args* a);
csa_status csa_index_topk(const csa_index_args* a, void* workspace, size_t workspace_bytes,
                          csa_stream_t stream);

/* csa_index_topk without a workspace argument.  (The pages have no
 * counterpart: this is a deployment variant of the call above.)
 * For callers that cannot allocate device memory on their hot path (a
 * runtime whose caching allocator already owns the GPU, or a loop that must
 * not call cudaMalloc because it may synchronise the device): the scratch is
 * a fixed 16 MiB array in the library's device image, held by every GPU that
 * loads the library until the process exits.
 *   - Same arguments and results as csa_index_topk.
 *   - Returns CSA_ERR_WORKSPACE, before any launch, when
 *     csa_index_workspace_size(a) > csa_index_noalloc_capacity().
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Every call on a device shares the array, which keeps the last call's
 *     contents (the kernels clear what must start at zero); calls that may
 *     overlap on the GPU (unordered streams) race on it.
 *   - Calls no cudaMalloc / cudaFree or allocating library routine. */
size_t csa_index_noalloc_capacity(void);
csa_status csa_index_topk_noalloc(const csa_index_args* a, csa_stream_t stream);

/* Top-K of given fp32 scores (same selection rule as csa_index_topk):
 * row b is scores + b*row_stride (elements), n values; idx is [B][K]. */
size_t csa_topk_workspace_size(int32_t B, int64_t n);
csa_status csa_topk_scores(const float* scores, int32_t B, int64_t n, int64_t row_stride,
                           int32_t K, int32_t* idx, void* workspace, size_t workspace_bytes,
                           csa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* (c) Sparse MLA attention.  For query t of sequence b and head h:
 *   entries = { dequant(kv entry idx[b,t,i]) : idx >= 0 }  followed by
 *             { dequant(window row t + r) : 0 <= r < n_win }   (duplicates kept)
 *   l_e  = softmax_scale * <q[b,t,h], x_e>
 *   out  = sum_e softmax(l, sink_h)_e * x_e ;  lse = log(sum_e exp(l_e) [+ exp(sink_h)])
 * x_e is all 512 latent channels (keys = values).  The window rows of
 * sequence b are at win + b*win_batch_stride + r*win_row_stride (528-B
 * entries); main entries at kv + b*kv_batch_stride + s*kv_row_stride (288 B).
 * Window entries are computed in fp16 and must decode to |x| < 65504. */
typedef struct {
  int32_t B, n_q, H, D;      /* H in {16, 32, 64}; D must be 512 */
  const float* q;            /* fp32 [B][n_q][H][D] */
  const uint8_t* kv;         /* FP4 main-KV entries */
  int64_t kv_row_stride;     /* bytes, >= 288, multiple of 16 */
  int64_t kv_batch_stride;   /* bytes, multiple of 16 */
  const int32_t* idx;        /* int32 [B][n_q][K], -1 = no entry */
  int32_t K;                 /* 0..65536 */
  const uint8_t* win;        /* FP8 window entries (may be NULL when n_win = 0) */
  int64_t win_row_stride;    /* bytes, >= 528, multiple of 16 */
  int64_t win_batch_stride;  /* bytes, multiple of 16 */
  int32_t n_win;             /* window entries per query, 0..1024 */
  float softmax_scale;
  const float* sink;         /* optional fp32 [H] sink logits */
  float* out;                /* fp32 [B][n_q][H][D] (bf16 with out_bf16) */
  float* lse;                /* optional fp32 [B][n_q][H] (natural log) */
  /* Partial RoPE around the attention (DeepSeek-V4.1-Flash architecture
   * database: "partial RoPE (last 64 dims of Q and KV; inverse rotation on
   * attention output)"; Model techniques map: fused RoPE-attention-RoPE-cast
   * kernel).  Optional fp32 [B][n_q][32][2]: (cos, sin) of the 32 angles of
   * query t's position.  When given, channels (448 + 2i, 449 + 2i) of q are
   * rotated by angle i (x + iy times e^{i angle}) before the logits and the
   * same channels of out are rotated back (angle negated); the cached
   * entries are taken as already rotated.  NULL = no rotation. */
  const float* rope_cs;
  int32_t out_bf16;          /* 1: out is bf16 [B][n_q][H][D], round to nearest even */
} csa_attn_args;

size_t csa_attn_workspace_size(const csa_attn_args* a);
csa_status csa_sparse_attn(const csa_attn_args* a, void* workspace, size_t workspace_bytes,
                           csa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* A stack of layers, one decode (or prefill) step.
 *   FULL    : encode `append` rows, index.* scoring + Top-K (+ pool build),
 *             then attention with attn.idx = index.idx.
 *   REINDEX : as FULL (index.keys and attn.kv normally point at the owner
 *             layer's caches); with pool_from >= 0, index.pool / pool_len /
 *             pool_cap are taken from layer pool_from's pool_out.
 *   REUSE   : no scoring; attention with attn.idx = the idx of layer
 *             reuse_from (attn.K likewise).
 *   SWA     : no scoring; attention over the window alone (attn.K = 0).
 * `append[i]` with src != NULL encodes new rows (e.g. this step's token)
 * into the caches before any layer's scoring (all appends of the stack run
 * first, in one launch).
 *
 * Ordering: the result is as if the layers ran in order on `stream`.
 * Internally, layers that do not depend on each other run concurrently on
 * auxiliary streams that the library creates once per device (no device
 * memory). Each auxiliary stream forks from `stream` by event and is joined
 * back into `stream` before the call returns, also when a launch fails part
 * way. Work enqueued on `stream` afterwards therefore sees every output, and
 * a stream capture of the call records the fork and join as graph edges.
 * Calls from several host threads are allowed: enqueues on one device are
 * serialised by a lock. */
typedef struct {
  const void* src;           /* NULL = no job */
  int32_t src_dtype;
  int32_t dim;
  int64_t n_rows;
  int64_t src_row_stride;    /* elements */
  int32_t fmt;
  void* dst;
  int64_t dst_row_stride;    /* bytes */
} csa_quant_job;

typedef struct {
  int32_t mode;              /* csa_mode */
  int32_t reuse_from;        /* REUSE: earlier layer index */
  int32_t pool_from;         /* REINDEX: earlier layer that built a pool, or -1 */
  csa_quant_job append[3];
  csa_index_args index;      /* unused for REUSE */
  csa_attn_args attn;        /* attn.idx / attn.K are filled in by the step */
} csa_layer_desc;

size_t csa_layer_workspace_size(const csa_layer_desc* layers, int32_t n_layers);
csa_status csa_layer_step(const csa_layer_desc* layers, int32_t n_layers, void* workspace,
                          size_t workspace_bytes, csa_stream_t stream);

/* csa_layer_step with hooks for overlapping host <-> device transfers with
 * the step (no counterpart on the pages; a serving loop's copies).  Every
 * field may be NULL; events are cudaEvent_t of the stream's device.
 *   queries_ready : the step reads the layers' attention queries (attn.q)
 *                   only after this event completes, so their upload may
 *                   still be in flight on another stream when the call is
 *                   made.  Everything else (appended rows, index queries and
 *                   weights, caches) must be ready as for csa_layer_step.
 *   layer_done[i] : recorded once layer i's outputs (attn.out, attn.lse and,
 *                   for an indexing layer, index.idx) are written, so that
 *                   their download can start while later layers still run.
 * Ordering on `stream` is as for csa_layer_step (the call's end on `stream`
 * follows every layer). */
typedef struct {
  void* queries_ready;
  void* layer_done[64];
} csa_step_sync;
csa_status csa_layer_step_sync(const csa_layer_desc* layers, int32_t n_layers, void* workspace,
                               size_t workspace_bytes, const csa_step_sync* sync, csa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Opt-in timing of the library's own kernels (profiling support, no
 * counterpart on the pages).  While enabled, each kernel launch is bracketed
 * by two CUDA events recorded on its launch stream.  csa_profile_collect()
 * waits for the recorded events, writes up to max_entries per-kernel totals
 * (name, launches, summed milliseconds) and forgets them; it returns the
 * number of distinct kernel names seen. */
typedef struct {
  char name[56];
  uint64_t launches;
  double total_ms;
} csa_kernel_time;
int32_t csa_profile_enable(int32_t on);   /* returns the previous state */
int32_t csa_profile_collect(csa_kernel_time* out, int32_t max_entries);
/* Launches recorded while a stream was being captured into a CUDA graph
 * become external event-record nodes, recorded again by every replay:
 * csa_profile_snapshot() reads the current totals without forgetting the
 * records (call it after each replay); csa_profile_reset() forgets them. */
int32_t csa_profile_snapshot(csa_kernel_time* out, int32_t max_entries);
void csa_profile_reset(void);

/* ------------------------------------------------------------------------ */
/* Context-parallel decode of one long sequence.  The positions [0, T) are
 * split into contiguous shards [t0, t1), one per rank, in rank order; each
 * rank holds its shard's keys and main KV, the last rank also the window.
 * The pages give no multi-GPU scheme; these kernels follow from the Top-K
 * rule and the softmax of the calls above (Model techniques map,
 * "Indexer-selected sparse attention" and "Multi-head latent attention"
 * rows).  A decode step:
 *   1. csa_index_topk on the shard (T = t1 - t0, scores requested), then
 *      csa_cp_local_pairs: the shard's Top-K as (score, global position);
 *   2. all-gather of the pairs over the ranks (caller: NCCL), rank-major
 *      [R][B][K_local];
 *   3. csa_cp_merge_topk: the global Top-K [B][K] (exact: every global
 *      winner is among its shard's K best; ties to the lower position);
 *   4. csa_cp_localize to this shard, csa_sparse_attn over it (sink NULL;
 *      the window only on the last rank) -> (out_r, lse_r);
 *   5. all-gather of (out_r, lse_r), rank-major; csa_cp_combine.
 * All pointers are device pointers; every call is asynchronous on `stream`. */
/* idx: [B][K] shard-local positions (-1 = none); scores: [B][score_stride]
 * the shard's scores; writes pair_score / pair_pos [B][K] = (scores[b][p],
 * p + t0), or (-inf, -1) for padding. */
csa_status csa_cp_local_pairs(const int32_t* idx, const float* scores, int32_t B, int32_t K, int64_t score_stride,
                              int64_t t0, float* pair_score, int32_t* pair_pos, csa_stream_t stream);
/* pair_score / pair_pos: [R][B][K_local] gathered in rank order (each list
 * ascending with trailing -1); idx: out [B][K] ascending positions, -1
 * padded.  R <= 1024. */
size_t csa_cp_merge_workspace_size(int32_t R, int32_t B, int32_t K_local);
csa_status csa_cp_merge_topk(const float* pair_score, const int32_t* pair_pos, int32_t R, int32_t B,
                             int32_t K_local, int32_t K, int32_t* idx, void* workspace, size_t workspace_bytes,
                             csa_stream_t stream);
/* idx_local[i] = idx[i] - t0 for idx[i] in [t0, t1), else -1 ([B][K]). */
csa_status csa_cp_localize(const int32_t* idx, int32_t B, int32_t K, int64_t t0, int64_t t1, int32_t* idx_local,
                           csa_stream_t stream);
/* o_parts [R][B][H][512], lse_parts [R][B][H] (natural log; -inf for a rank
 * with no entries); sink optional [H]; out [B][H][512], lse optional [B][H]. */
csa_status csa_cp_combine(const float* o_parts, const float* lse_parts, int32_t R, int32_t B, int32_t H,
                          const float* sink, float* out, float* lse, csa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Measurement kernels (no counterpart on the pages, which report no hardware
 * figure): the roofline denominators, measured in the same run as the kernels
 * they judge.
 * csa_bench_copy: copy `bytes` (a multiple of 16; both pointers 16-byte
 *   aligned) from src to dst with 128-bit loads and stores; HBM traffic is
 *   2 * bytes.  CSA_ERR_ALIGNMENT otherwise.
 * csa_bench_fp8_gemm: D[M][N] (fp32, row-major) = A[M][K] * B[N][K]^T with
 *   A and B E4M3 bytes, row-major (K contiguous), on the tcgen05 tensor cores;
 *   M a multiple of 128, N of 256, K of 128 (CSA_ERR_SHAPE otherwise);
 *   2*M*N*K flops. */
csa_status csa_bench_copy(const void* src, void* dst, size_t bytes, csa_stream_t stream);
csa_status csa_bench_fp8_gemm(const uint8_t* A, const uint8_t* B, float* D, int32_t M, int32_t N, int32_t K,
                              csa_stream_t stream);

/* ------------------------------------------------------------------------ */
const char* csa_status_string(int32_t status);
/* Device-side error code recorded by a kernel whose bounded wait on an
 * mbarrier timed out (0 = none), then cleared.  Synchronises with the device
 * (it copies the flag back); call it after the work it should cover. */
int32_t csa_device_status(void);
/* Number of kernels the library has enqueued since load (all entry points). */
uint64_t csa_launch_count(void);
int32_t csa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
