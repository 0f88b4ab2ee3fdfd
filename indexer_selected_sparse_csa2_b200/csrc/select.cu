// Exact Top-K selection (lowest-position tie-break, ascending output).
//
// Selection rule of the lightning indexer (Model techniques map -
// DeepSeek-V4.1-Flash, "Indexer-selected sparse attention" row: each query
// attends only to the index_topk best-scored tokens).  Ties are broken
// towards the lower position so the result is one well-defined set.
//
// Three stages over rows of fp32 values (order_key maps them to uint32 keys
// that sort like the values):
//   hist    - 4096-bin histogram of key >> 20 per row (usually fused into the
//             producer of the values, e.g. the indexer scoring kernel);
//   extract - many CTAs per row: find the bin b1 holding the K-th largest key,
//             then copy every slot whose bin is >= b1 into that CTA's own
//             region of a candidate buffer, in slot order, plus a count;
//   final   - one CTA per row: concatenate the candidate runs (still in slot
//             order), run an 8-bit radix select on the full 32-bit key to get
//             the exact K-th key tau and how many slots equal to tau are
//             needed, then emit the selected slots in slot order (so the
//             output is ascending and the lowest equal slots win).
#include "select.cuh"

namespace csa {

constexpr int kExtractThreads = 256;     // 8 warps = 8 consecutive runs per CTA
constexpr int kRunsPerCta = kExtractThreads / 32;
constexpr int kFinalThreads = 1024;
constexpr int kListCap = 20480;          // candidates staged in shared memory
constexpr int kMaxRuns = 8192;
constexpr int kRunsPerThread = kMaxRuns / kFinalThreads;

struct SelectJobs {
  SelectJob j[2];
};

SelectPlan plan_select(int B, int64_t n) {
  SelectPlan p;
  // about four resident extract CTAs per SM over all rows; each warp scans
  // one run of at least 512 slots; at most kMaxRuns runs per row.
  int64_t ctas = ((int64_t)kNumSMs * 4 + B - 1) / (B > 0 ? B : 1);
  if (ctas < 1) ctas = 1;
  int64_t run = (n + ctas * kRunsPerCta - 1) / (ctas * kRunsPerCta);
  if (run < 512) run = 512;
  const int64_t minr = (n + kMaxRuns - 1) / kMaxRuns;
  if (run < minr) run = minr;
  run = (run + 127) / 128 * 128;
  p.chunk = run;
  p.nchunks = (int)((n + run - 1) / run);
  if (p.nchunks < 1) p.nchunks = 1;
  return p;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t select_workspace_bytes(int B, int64_t n) {
  SelectPlan p = plan_select(B, n);
  size_t s = 0;
  s += align256((size_t)B * kHistBins * 4);
  s += 4 * align256((size_t)B * (size_t)(n > 0 ? n : 1) * 4);
  s += align256((size_t)B * p.nchunks * 4);
  return s;
}

size_t select_carve(SelectJob& j, int B, int64_t n, void* ws) {
  SelectPlan p = plan_select(B, n);
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = 0;
  const size_t nn = (size_t)(n > 0 ? n : 1);
  j.hist = reinterpret_cast<uint32_t*>(base + off); off += align256((size_t)B * kHistBins * 4);
  j.cand_key = reinterpret_cast<uint32_t*>(base + off); off += align256((size_t)B * nn * 4);
  j.cand_pos = reinterpret_cast<int32_t*>(base + off); off += align256((size_t)B * nn * 4);
  j.list_key = reinterpret_cast<uint32_t*>(base + off); off += align256((size_t)B * nn * 4);
  j.list_pos = reinterpret_cast<int32_t*>(base + off); off += align256((size_t)B * nn * 4);
  j.cnt = reinterpret_cast<int32_t*>(base + off); off += align256((size_t)B * p.nchunks * 4);
  j.chunk = p.chunk;
  j.nchunks = p.nchunks;
  j.n = n;
  return off;
}

// ------------------------------------------------------------------ zero --
__global__ void zero_kernel(uint4* p, size_t n16) {
  pdl_enter();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    p[i] = make_uint4(0, 0, 0, 0);
}

cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t stream) {
  size_t n16 = bytes / 16;
  if (n16 == 0) return cudaSuccess;
  int g = (int)((n16 + 255) / 256);
  if (g > kNumSMs * 8) g = kNumSMs * 8;
  ProfScope ps(stream, "zero");
  launch_k(zero_kernel, dim3(g), dim3(256), 0, stream, static_cast<uint4*>(p), n16);
  note_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ hist --
__global__ void __launch_bounds__(256) select_hist_kernel(SelectJobs jobs) {
  pdl_enter();
  const SelectJob& J = jobs.j[blockIdx.z];
  const int b = blockIdx.y;
  const int c = blockIdx.x;
  if (c * kRunsPerCta >= J.nchunks) return;
  __shared__ uint32_t h[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t nrow = J.n_row ? (int64_t)min((int64_t)J.n_row[b], J.n) : J.n;
  const int64_t lo = (int64_t)c * kRunsPerCta * J.chunk;
  const int64_t hi = min(lo + kRunsPerCta * J.chunk, nrow);
  const float* v = J.vals + (int64_t)b * J.row_stride;
  for (int64_t s = lo + threadIdx.x; s < hi; s += blockDim.x) atomicAdd(&h[order_key(v[s]) >> (32 - kHistBits)], 1u);
  __syncthreads();
  uint32_t* g = J.hist + (int64_t)b * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

// -------------------------------------------------------------- block scan --
// Inclusive scan over the block (blockDim.x multiple of 32, <= 1024).
template <int NT>
CSA_DEV uint32_t block_incl_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) warp_tot[wid] = v;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < NT / 32 ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < NT / 32) warp_tot[lane] = w;
    if (lane == NT / 32 - 1) *total = w;
  }
  __syncthreads();
  const uint32_t r = v + (wid > 0 ? warp_tot[wid - 1] : 0u);
  __syncthreads();
  return r;
}

// Find the first-level threshold bin: the largest bin beta with
// sum_{bins >= beta} >= K (0 when the row holds fewer than K values).
// Called by all NT threads of the block.
template <int NT>
CSA_DEV int threshold_bin(const uint32_t* gh, int K, uint32_t* warp_tot, uint32_t* total, int* out_bin) {
  // thread i covers bins [PB*(NT-1-i), PB*(NT-1-i)+PB): scanning threads in
  // order walks the bins from the top down.
  constexpr int PB = kHistBins / NT;
  static_assert(PB * NT == kHistBins, "layout");
  const int i = threadIdx.x;
  uint32_t loc[PB];
  uint32_t s = 0;
  const int base = PB * (NT - 1 - i);
#pragma unroll
  for (int k = 0; k < PB; ++k) { loc[k] = gh[base + k]; s += loc[k]; }
  if (i == 0) *out_bin = 0;
  const uint32_t incl = block_incl_scan<NT>(s, warp_tot, total);
  const uint32_t excl = incl - s;
  if (excl < (uint32_t)K && incl >= (uint32_t)K) {
    uint32_t cum = excl;
    for (int k = PB - 1; k >= 0; --k) {
      cum += loc[k];
      if (cum >= (uint32_t)K) { *out_bin = base + k; break; }
    }
  }
  __syncthreads();
  return *out_bin;
}

// Each warp scans one run of slots in order, 4 slots per lane per step, and
// appends the run's candidates (bin >= beta) to the run's own region of the
// candidate buffer, keeping slot order (lane-order prefix via shuffles).
template <bool VEC>
__global__ void __launch_bounds__(kExtractThreads) select_extract_kernel(SelectJobs jobs) {
  pdl_enter();
  const SelectJob& J = jobs.j[blockIdx.z];
  const int b = blockIdx.y;
  if ((int)blockIdx.x * kRunsPerCta >= J.nchunks) return;
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t total;
  __shared__ int bin;
  const int beta = threshold_bin<kExtractThreads>(J.hist + (int64_t)b * kHistBins, J.K, warp_tot, &total, &bin);
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kRunsPerCta + (threadIdx.x >> 5);
  if (r >= J.nchunks) return;
  const int64_t nrow = J.n_row ? (int64_t)min((int64_t)J.n_row[b], J.n) : J.n;
  const int64_t lo = (int64_t)r * J.chunk;
  const int64_t hi = min(lo + J.chunk, nrow);
  const float* v = J.vals + (int64_t)b * J.row_stride;
  uint32_t* ck = J.cand_key + (int64_t)b * J.n + lo;
  int32_t* cp = J.cand_pos + (int64_t)b * J.n + lo;
  uint32_t run = 0;
  for (int64_t s0 = lo; s0 < hi; s0 += 128) {
    const int64_t s = s0 + 4 * lane;
    float x[4];
    if (VEC && s + 3 < hi) {
      const float4 f = *reinterpret_cast<const float4*>(v + s);
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = s + k < hi ? v[s + k] : 0.f;
    }
    uint32_t key[4];
    uint32_t flags = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      key[k] = order_key(x[k]);
      if (s + k < hi && (int)(key[k] >> (32 - kHistBits)) >= beta) flags |= 1u << k;
    }
    const uint32_t c = __popc(flags);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t at = run + incl - c;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (flags & (1u << k)) {
        ck[at] = key[k];
        cp[at] = (int32_t)(s + k);
        ++at;
      }
    }
    run += tot;
  }
  if (lane == 0) J.cnt[(int64_t)b * J.nchunks + r] = (int32_t)run;
}

// ----------------------------------------------------------------- final --
CSA_DEV void write_selected(const SelectJob& J, int b, uint32_t j, int32_t slot) {
  int32_t* out = J.out + (int64_t)b * J.out_stride;
  int32_t pos = J.map ? J.map[(int64_t)b * J.map_stride + slot] : slot;
  if (J.expand == 0) {
    out[j] = pos;
  } else {
    for (int r = 0; r < J.expand; ++r) {
      int64_t p = (int64_t)pos * J.expand + r;
      out[(int64_t)j * J.expand + r] = p < J.limit ? (int32_t)p : -1;
    }
  }
}

__global__ void __launch_bounds__(kFinalThreads, 1) select_final_kernel(SelectJobs jobs) {
  pdl_enter();
  const SelectJob& J = jobs.j[blockIdx.y];
  const int b = blockIdx.x;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* offs = reinterpret_cast<uint32_t*>(smem);                       // [kMaxRuns]
  uint32_t* skey = offs + kMaxRuns;                                          // [kListCap]
  int32_t* spos = reinterpret_cast<int32_t*>(skey + kListCap);               // [kListCap]
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t total;
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_krem;
  const int tid = threadIdx.x;
  const int nruns = J.nchunks;
  const int32_t* cnt_row = J.cnt + (int64_t)b * nruns;

  // 1. run offsets (thread t owns runs [8t, 8t + 8))
  uint32_t c8[kRunsPerThread];
  uint32_t mine = 0;
#pragma unroll
  for (int k = 0; k < kRunsPerThread; ++k) {
    const int r = kRunsPerThread * tid + k;
    c8[k] = r < nruns ? (uint32_t)cnt_row[r] : 0u;
    mine += c8[k];
  }
  const uint32_t incl = block_incl_scan<kFinalThreads>(mine, warp_tot, &total);
  const uint32_t m = total;
  {
    uint32_t o = incl - mine;
#pragma unroll
    for (int k = 0; k < kRunsPerThread; ++k) {
      offs[kRunsPerThread * tid + k] = o;
      o += c8[k];
    }
  }
  __syncthreads();

  // 2. contiguous ordered list (shared memory when it fits).  List element i
  //    comes from the last run r with offs[r] <= i (a binary search over the
  //    run offsets; runs past nruns hold offset m); each thread moves four
  //    elements per round so their loads are in flight together.
  const bool in_smem = m <= (uint32_t)kListCap;
  uint32_t* lk = in_smem ? skey : J.list_key + (int64_t)b * J.n;
  int32_t* lp = in_smem ? spos : J.list_pos + (int64_t)b * J.n;
  {
    const uint32_t* ck = J.cand_key + (int64_t)b * J.n;
    const int32_t* cp = J.cand_pos + (int64_t)b * J.n;
    for (uint32_t i0 = tid; i0 < m; i0 += 4 * kFinalThreads) {
      int64_t src[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t i = i0 + u * kFinalThreads;
        int r = 0;   // invariant offs[r] <= i; r + step <= kMaxRuns - 1 at every step
#pragma unroll
        for (int step = kMaxRuns / 2; step >= 1; step >>= 1)
          if (offs[r + step] <= i) r += step;
        src[u] = (int64_t)r * J.chunk + (i - offs[r]);
      }
      uint32_t kk[4];
      int32_t pp[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t i = i0 + u * kFinalThreads;
        if (i < m) { kk[u] = ck[src[u]]; pp[u] = cp[src[u]]; }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t i = i0 + u * kFinalThreads;
        if (i < m) { lk[i] = kk[u]; lp[i] = pp[u]; }
      }
    }
  }
  __syncthreads();

  // 3. exact threshold tau by 4 passes of an 8-bit radix select, and the
  //    number of slots equal to tau that the Top-K still needs
  const uint32_t K = (uint32_t)J.K;
  const bool take_all = m <= K;
  if (tid == 0) { s_prefix = 0; s_krem = K; }
  __syncthreads();
  if (!take_all) {
    uint32_t mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kFinalThreads) hist[i] = 0;
      __syncthreads();
      const uint32_t prefix = s_prefix;
      for (uint32_t i = tid; i < m; i += kFinalThreads) {
        const uint32_t k = lk[i];
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // lane l covers digits [255-8l-7, 255-8l], scanning from the top
        uint32_t loc[8];
        uint32_t s = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) { loc[k] = hist[255 - 8 * tid - k]; s += loc[k]; }
        uint32_t inc = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
          if (tid >= o) inc += t;
        }
        const uint32_t exc = inc - s;
        const uint32_t krem = s_krem;
        if (exc < krem && inc >= krem) {
          uint32_t cum = exc;
          for (int k = 0; k < 8; ++k) {
            if (cum + loc[k] >= krem) {
              const uint32_t d = 255u - 8u * tid - k;
              s_prefix = prefix | (d << shift);
              s_krem = krem - cum;
              break;
            }
            cum += loc[k];
          }
        }
      }
      mask |= 255u << shift;
      __syncthreads();
    }
  }
  const uint32_t tau = s_prefix;
  const uint32_t need_eq = s_krem;   // slots equal to tau to take, lowest first

  // 4. ordered emission: thread t owns the contiguous segment
  //    [t*seg, (t+1)*seg) of the list
  const uint32_t seg = (m + kFinalThreads - 1) / kFinalThreads;
  const uint32_t i0 = min(m, tid * seg), i1 = min(m, i0 + seg);
  uint32_t n_eq = 0;
  if (!take_all)
    for (uint32_t i = i0; i < i1; ++i) n_eq += lk[i] == tau ? 1u : 0u;
  const uint32_t eq_excl = block_incl_scan<kFinalThreads>(n_eq, warp_tot, &total) - n_eq;
  uint32_t n_sel = 0;
  {
    uint32_t eq_rank = eq_excl;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint32_t k = lk[i];
      bool sel = take_all || k > tau;
      if (!take_all && k == tau) { sel = eq_rank < need_eq; ++eq_rank; }
      n_sel += sel ? 1u : 0u;
    }
  }
  const uint32_t sel_incl = block_incl_scan<kFinalThreads>(n_sel, warp_tot, &total);
  const uint32_t out_count = total;
  {
    uint32_t j = sel_incl - n_sel;
    uint32_t eq_rank = eq_excl;
    for (uint32_t i = i0; i < i1; ++i) {
      const uint32_t k = lk[i];
      bool sel = take_all || k > tau;
      if (!take_all && k == tau) { sel = eq_rank < need_eq; ++eq_rank; }
      if (sel) write_selected(J, b, j++, lp[i]);
    }
  }

  // 5. padding and valid length
  const int32_t width = J.out_width;
  int32_t* out = J.out + (int64_t)b * J.out_stride;
  const int64_t written = (int64_t)out_count * (J.expand ? J.expand : 1);
  for (int64_t j = written + tid; j < width; j += kFinalThreads) out[j] = -1;
  __syncthreads();
  if (J.expand && J.out_len && tid == 0) {
    // only the highest selected block can reach past the limit
    int64_t bad = 0;
    for (int64_t j = written - J.expand; j < written; ++j)
      if (j >= 0 && out[j] < 0) ++bad;
    J.out_len[b] = (int32_t)(written - bad);
  }
}

cudaError_t launch_hist_only(const float* vals, int64_t row_stride, int64_t n, const int32_t* n_row,
                             uint32_t* hist, int B, cudaStream_t stream) {
  SelectJobs js;
  SelectPlan p = plan_select(B, n);
  SelectJob& j = js.j[0];
  j = SelectJob{};
  j.vals = vals;
  j.row_stride = row_stride;
  j.n = n;
  j.n_row = n_row;
  j.hist = hist;
  j.chunk = p.chunk;
  j.nchunks = p.nchunks;
  js.j[1] = j;
  dim3 g((p.nchunks + kRunsPerCta - 1) / kRunsPerCta, B, 1);
  ProfScope ps(stream, "select_hist");
  launch_k(select_hist_kernel, dim3(g), dim3(256), 0, stream, js);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectJob* jobs, int njobs, int B, bool build_hist, cudaStream_t stream) {
  SelectJobs js;
  js.j[0] = jobs[0];
  js.j[1] = njobs > 1 ? jobs[1] : jobs[0];
  int maxc = 0;
  bool vec = true;
  for (int i = 0; i < njobs; ++i) {
    const int ctas = (jobs[i].nchunks + kRunsPerCta - 1) / kRunsPerCta;
    maxc = ctas > maxc ? ctas : maxc;
    vec = vec && (((uintptr_t)jobs[i].vals & 15) == 0) && (jobs[i].row_stride % 4 == 0);
  }
  dim3 g(maxc, B, njobs);
  if (build_hist) {
    ProfScope ps(stream, "select_hist");
    launch_k(select_hist_kernel, dim3(g), dim3(256), 0, stream, js);
    note_launches(1);
  }
  {
    ProfScope ps(stream, "select_extract");
    if (vec) launch_k(select_extract_kernel<true>, dim3(g), dim3(kExtractThreads), 0, stream, js);
    else launch_k(select_extract_kernel<false>, dim3(g), dim3(kExtractThreads), 0, stream, js);
  }
  const size_t smem = (size_t)kMaxRuns * 4 + (size_t)kListCap * 8;
  static SmemAttrOnce attr;
  const cudaError_t ea = attr.set(select_final_kernel, smem);
  if (ea != cudaSuccess) return ea;
  {
    ProfScope ps(stream, "select_final");
    launch_k(select_final_kernel, dim3(dim3(B, njobs)), dim3(kFinalThreads), smem, stream, js);
  }
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace csa
