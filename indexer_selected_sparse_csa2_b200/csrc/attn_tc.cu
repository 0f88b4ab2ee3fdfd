// Sparse MLA attention on the 5th-generation tensor cores (tcgen05), built
// for 64 query heads (the shape of the step's attention layers); 16 or 32
// heads run the same kernel with the query rows of heads >= H left zero and
// only heads < H written.
//
// Same function as sparse_attn_mma_kernel (MLA over the Top-K selected FP4
// entries plus the FP8 window, K = V = the 512-wide latent; Model techniques
// map - DeepSeek-V4.1-Flash, "Multi-head latent attention", "Indexer-selected
// sparse attention", "Sliding-window attention" and "Learnable attention
// sink" rows).  Per 64-entry tile of one token:
//   S2 = Q2 K^T   tcgen05.mma kind::f16, M = 128 rows of Q2: row 2h is the
//                 fp16 hi part of head h's query, row 2h+1 the lo part
//                 fp16(q - hi); N = 64 entries, K = 512; fp32 in TMEM.  The
//                 first 384 channels of Q2 stay in TMEM as the A operand
//                 (no shared-memory traffic for them), the last 128 in
//                 shared memory.  The softmax adds the two rows of a head
//                 (neighbouring lanes of one warp), which carries ~22 bits of
//                 q against the exactly dequantised fp16 entries.
//   O^T += V^T P^T  tcgen05.mma kind::f16, M = 128 latent channels (4
//                 chunks), N = 64 heads, K = 64 entries, fp32 in TMEM, once
//                 for the fp16 hi part of P and once for the lo part.  The
//                 same shared-memory tile of dequantised entries is the
//                 K-major B operand of S2 and the MN-major A operand here.
// Warp roles: warps 0-3 softmax / output (one TMEM lane quarter each; the
// two lanes of a head split the tile's entries), warps 4-11 gather +
// dequantise (8 lanes take 8 entries, 4 lanes per entry, 128 channels each;
// the codes of the next tile's entries are staged by cp.async into each
// lane's own 128-byte shared-memory slot, and their block scales loaded,
// while the current tile is decoded), warp 12 issues the S2 MMAs, warp 13 the
// PV MMAs.  Entry
// tiles and P are double buffered, so tile i+1 is dequantised while S2, the
// softmax and PV of tile i run.  Online softmax in the exp2 domain with lazy
// rescaling: the running max only moves when a tile's max exceeds it by more
// than 8, and only then are the O^T accumulators rescaled in TMEM.
//
// Channel order: inside every group of 8 channels the staged operands hold
// channels (0, 4, 1, 5, 2, 6, 3, 7), so one 32-bit word of FP4 codes turns
// into four fp16 pairs with shifts and masks only.  Q2 uses the same order
// (the dot products are unchanged) and the output un-permutes O^T's rows.
// Main (FP4) entries are staged as E2M1 * s * 2^-7 (exact in fp16, one
// multiply per channel pair); their logits are scaled by 2^7 and their
// probabilities by 2^7 in P, which leaves S and O unchanged.  Window entries
// are staged unscaled.
//
// With several splits per token the partial O^T (unnormalised) is written
// from TMEM to global memory as [head][channel] fp32 rows (coalesced per
// head); attn_combine merges the splits.  The kernel triggers its dependents at once and does its prologue
// (barrier setup, TMEM allocation, the query staging from caller memory or
// from the stack's staging buffer, which a full event dependency orders)
// before it waits for the previous kernel on its stream, so the prologue
// overlaps that kernel's tail.  All waits are bounded (sm100.cuh).
#include "sm100.cuh"
#include "q2.cuh"
#include "attn_tc.cuh"
#include "rope.cuh"

namespace csa {

constexpr int kAtH = 64;                  // heads
constexpr int kAtE = 64;                  // entries per tile
constexpr int kAtDeqWarps = 8;
constexpr int kAtWarpS = 4 + kAtDeqWarps;           // S2 issuer
constexpr int kAtWarpPV = kAtWarpS + 1;             // PV issuer
constexpr int kAtThreads = 32 * (kAtWarpPV + 1);    // 448
constexpr int kAtQTmemBlocks = 6;                   // 64-channel blocks of Q2 in TMEM
constexpr int kAtQSmemBlocks = 8 - kAtQTmemBlocks;  // ... and in shared memory
constexpr int kAtQBlkBytes = 128 * 128;             // 128 rows x 64 fp16
constexpr int kAtKVBlk = kAtE * 128;                // one 64-channel block of an entry tile
constexpr int kAtKVBytes = 8 * kAtKVBlk;            // 64 KB
constexpr int kAtPBytes = kAtH * kAtE * 2;          // P^T part (hi or lo): 64 head rows x 128 B
constexpr int kAtRawBytes = 256 * 128;            // cp.async staging: one 128-byte slot per gather thread
constexpr size_t kAtSmemBytes =
    1024 + (size_t)kAtQSmemBlocks * kAtQBlkBytes + 2 * kAtKVBytes + 4 * kAtPBytes + kAtRawBytes + 1024;
constexpr uint32_t kAtTmemCols = 512;
constexpr uint32_t kAtSCol = 32 * kAtQTmemBlocks;   // S2: 64 fp32 columns after Q2
constexpr uint32_t kAtOCol = 256;                   // O^T chunk c: columns 256 + 64c
static_assert(kAtSCol + kAtE <= kAtOCol, "TMEM map");
constexpr float kAtLog2e = 1.4426950408889634f;
constexpr float kAtLn2 = 0.6931471805599453f;
constexpr float kAtRescale = 8.0f;        // lazy-rescale threshold (exp2 units)

static __device__ int g_at_error;

struct AtSmem {
  uint8_t* q2;      // Q2 channels 384..511 (2 blocks)
  uint8_t* kv;      // 2 entry tiles
  uint8_t* p;       // 2 x (P^T hi, P^T lo)
  uint8_t* raw;     // [256 gather threads][128 B] staged entry codes
  float* scl;       // [64] per-head output scale
  float* alpha_s;   // [2][64] by tile parity (a warp may run one tile ahead)
  int* o_bad;       // O^T not valid (a wait gave up)
  uint64_t* bars;
  uint32_t* tmem_base;
};

CSA_DEV AtSmem carve_at(uint8_t* raw) {
  AtSmem s;
  uintptr_t base = (reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  s.q2 = p; p += kAtQSmemBlocks * kAtQBlkBytes;
  s.kv = p; p += 2 * kAtKVBytes;
  s.p = p; p += 4 * kAtPBytes;
  s.raw = p; p += kAtRawBytes;
  s.scl = reinterpret_cast<float*>(p); p += 64 * 4;
  s.alpha_s = reinterpret_cast<float*>(p); p += 2 * 64 * 4;
  s.o_bad = reinterpret_cast<int*>(p); p += 16;
  s.bars = reinterpret_cast<uint64_t*>(p); p += 16 * 8;
  s.tmem_base = reinterpret_cast<uint32_t*>(p);
  return s;
}

CSA_DEV uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
CSA_DEV __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Integer-pipe decoders (the conversion pipe is the scarce one here).
// An 8-bit E4M3 code c at bits 0-7 (and 16-23) becomes the fp16 value
// E4M3(c) * 2^-8 by moving exponent and mantissa up by 7 and the sign to bit
// 15; E4M3 subnormals land on fp16 subnormals, so every code is exact.  Bits
// 8-15 and 24-31 of t are ignored.
CSA_DEV uint32_t e4m3x2_bits_m8(uint32_t t) {
  return ((t << 7) & 0x3F803F80u) | ((t << 8) & 0x80008000u);
}
// The FP4 codes of channels kk and kk+4 of a word of 8 codes (channel c in
// bits 4c..4c+3) as fp16 E2M1 * 2^-14: the E2M1 magnitude bits go to fp16
// bits 9-11 (its exponent field lines up with the low fp16 exponent bits and
// its subnormal 0.5 with the fp16 subnormal 2^-15), the sign to bit 15.
template <int kk>
CSA_DEV uint32_t e2m1_pair_m14(uint32_t w) {
  const uint32_t mag = kk < 3 ? (w << (9 - 4 * kk)) : (w >> 3);
  const uint32_t sgn = w << (12 - 4 * kk);
  return (mag & 0x0E000E00u) | (sgn & 0x80008000u);
}
constexpr uint32_t kH2Exp15 = 0x78007800u;   // fp16x2 {2^15, 2^15}
CSA_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Bounded wait taken by a whole warp; the result is the same in every lane, so
// the warp-collective TMEM accesses after it stay convergent on every path.
CSA_DEV bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int code) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_at_error, code));
}

__global__ void __launch_bounds__(kAtThreads, 1) sparse_attn_tc_kernel(AttnTcParams p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  AtSmem S = carve_at(smem_raw);
  uint64_t* kv_full = S.bars + 0;    // [2] dequant -> S2 issuer (8 warp arrivals)
  uint64_t* kv_free = S.bars + 2;    // [2] PV done: entry tile and P buffer reusable
  uint64_t* s_full = S.bars + 4;     // S2 in TMEM
  uint64_t* s_free = S.bars + 5;     // S2 read by the softmax (4 warp arrivals)
  uint64_t* p_full = S.bars + 6;     // [2] P written, O^T rescaled (4 warp arrivals)
  uint64_t* o_done = S.bars + 8;     // one phase per PV
  uint64_t* drain = S.bars + 9;      // [2] all MMAs of an issuer retired (teardown; [1] = every PV, for the output)
  uint64_t* q_full = S.bars + 11;    // staged query copied in by the bulk copies
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bt = blockIdx.y;
  const int b = bt / p.n_q, tq = bt - b * p.n_q;
  const int split = blockIdx.x;
  const int n_tiles_all = (p.n_entries + kAtE - 1) / kAtE;
  const int tile0 = split * p.tiles_per_split;
  const int tile1 = min(tile0 + p.tiles_per_split, n_tiles_all);
  const int nt = max(0, tile1 - tile0);

  if (tid == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(kv_full + k, kAtDeqWarps);
      mbar_init(kv_free + k, 1);
      mbar_init(p_full + k, 4);
      mbar_init(drain + k, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(o_done, 1);
    mbar_init(q_full, 1);
    fence_mbar_init();
    *S.o_bad = 0;
    if (p.q2) {
      // the token's staged query: the tensor-memory part into the (still
      // idle) entry-tile buffers, the shared-memory part straight to its place
      const uint8_t* q2t = p.q2 + (size_t)(blockIdx.y) * kQ2TokenBytes;
      mbar_arrive_expect_tx(q_full, kQ2TokenBytes);
      for (int c = 0; c < kQ2TmemBytes; c += 32768) bulk_load(S.kv + c, q2t + c, 32768, q_full);
      bulk_load(S.q2, q2t + kQ2TmemBytes, kQ2SmemBytes, q_full);
    }
  }

  // gather role: 8 consecutive lanes take 8 different entries, so each
  // quarter-warp phase of a 16-byte shared store covers all 32 banks
  const int jd = tid - 128;
  const int e = 8 * (jd >> 5) + (jd & 7), q4 = (jd >> 3) & 3;   // entry, quarter (128 channels)
  const int32_t* idx_b = p.idx + (int64_t)bt * p.K;
  const uint8_t* kvb = p.kv + (int64_t)b * p.kv_batch_stride;
  const uint8_t* wb = p.win ? p.win + (int64_t)b * p.win_batch_stride : nullptr;
  uint2 rex = make_uint2(0, 0);
  int kind = 0;   // 0 invalid, 1 FP4 main entry, 2 FP8 window entry
  // this lane's staging slot; chunk k sits at chunk k ^ (jd & 7), so the
  // 8-lane groups of a warp read different banks
  const int swz = jd & 7;
  const uint32_t slot = smem_u32(S.raw) + 128u * (uint32_t)(jd & 255);
#define CSA_AT_FETCH(tile)                                                                                 \
  do {                                                                                                     \
    const int jj = (tile) * kAtE + e;                                                                      \
    kind = 0;                                                                                              \
    if (jj < p.K) {                                                                                        \
      const int pos = idx_b[jj];                                                                           \
      if (pos >= 0) {                                                                                      \
        const uint8_t* row = kvb + (int64_t)pos * p.kv_row_stride;                                         \
        _Pragma("unroll") for (int k = 0; k < 4; ++k) cp_async16(slot + 16u * (k ^ swz), row + 64 * q4 + 16 * k); \
        rex = *reinterpret_cast<const uint2*>(row + 256 + 8 * q4);                                         \
        kind = 1;                                                                                          \
      }                                                                                                    \
    } else if (jj < p.n_entries) {                                                                         \
      const uint8_t* row = wb + (int64_t)(tq + jj - p.K) * p.win_row_stride;                               \
      _Pragma("unroll") for (int k = 0; k < 8; ++k) cp_async16(slot + 16u * (k ^ swz), row + 128 * q4 + 16 * k); \
      rex.x = *reinterpret_cast<const uint32_t*>(row + 512 + 4 * q4);                                      \
      kind = 2;                                                                                            \
    }                                                                                                      \
    cp_async_commit();                                                                                     \
  } while (0)
  const bool is_deq = warp >= 4 && warp < kAtWarpS;
  // with the query staged by bulk copies the gather warps are free: the first
  // tile's loads go out now, under the staging
  if (p.q2 && is_deq && nt > 0) {
    pdl_wait();
    CSA_AT_FETCH(tile0);
  }

  if (warp == kAtWarpS) tmem_alloc(S.tmem_base, kAtTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *S.tmem_base;

  // ---- Q2 staging.  TMEM part (channels 0..383): TMEM column j of row
  // r = 2h + part holds the pair of channels (8g + (j & 3), 8g + (j & 3) + 4),
  // g = j / 4; lane quarter qq is written by warps qq, qq + 4 and qq + 8, four
  // 16-column stores each.
  const int H = p.H;                        // 16, 32 or 64 heads; rows of heads >= H stay zero
  const float* qg = p.q + (int64_t)bt * H * kD;
  if (p.q2) {
    // q staged by the stack prologue: copy rows into TMEM, the rest into shared memory
    // warps 0-3 (one TMEM lane quarter each) move the tensor-memory part
    // from shared memory into TMEM; the shared-memory part is already in place
    if (warp < 4) {
      const int r = 32 * warp + lane;
      if (!mbar_wait_warp(q_full, 0u, kErrWaitTmaFull)) {
        // leave the query unstaged (the error flag is set)
      } else {
        const uint4* row = reinterpret_cast<const uint4*>(S.kv + (size_t)r * kQ2TmemWords * 4);
#pragma unroll 1
        for (int c0 = 0; c0 < 48; c0 += 8) {            // 8 chunks = 32 columns per round
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 f = row[(c0 + k) ^ (r & 7)];
            v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
          }
          uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
          uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(v + 16);
          tmem_st16(tbase + ((uint32_t)(32 * warp) << 16) + 4u * c0, lo);
          tmem_st16(tbase + ((uint32_t)(32 * warp) << 16) + 4u * c0 + 16u, hi);
        }
        tmem_wait_st();
      }
    } else if (is_deq) {
      // the entry-tile buffers hold the staged query until the barrier below
    } else {
      mbar_wait_warp(q_full, 0u, kErrWaitTmaFull);     // S.q2 written before the MMAs read it
    }
  } else {
  if (warp < kAtWarpS) {
    const int qq = warp & 3, wr = warp >> 2;
    const int r = 32 * qq + lane, h = r >> 1;
    const bool lo = r & 1;
    const float4* qrow = reinterpret_cast<const float4*>(qg + (int64_t)(h < H ? h : 0) * kD);
#pragma unroll 1
    for (int u = 4 * wr; u < 4 * wr + 4; ++u) {         // columns 16u .. 16u + 15 = channels 32u .. 32u + 31
      float4 f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = h < H ? qrow[8 * u + k] : make_float4(0.f, 0.f, 0.f, 0.f);
      uint32_t v[16];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t o[4];
        q_hilo_perm8(f[2 * g], f[2 * g + 1], lo, o);
#pragma unroll
        for (int k = 0; k < 4; ++k) v[4 * g + k] = o[k];
      }
      tmem_st16(tbase + ((uint32_t)(32 * qq) << 16) + 16u * u, v);
    }
    tmem_wait_st();
  }
  // shared part (channels 384..511): two K-major 128-byte-swizzled blocks;
  // every load of a thread is issued before the first conversion
  {
    constexpr int kIt = (128 * 16 + kAtThreads - 1) / kAtThreads;
    float4 f[2 * kIt];
#pragma unroll
    for (int t = 0; t < kIt; ++t) {
      const int i = tid + t * kAtThreads;
      if (i < 128 * 16) {
        const int r = i >> 4, kb = (i >> 3) & 1, c8 = i & 7;
        const bool live = (r >> 1) < H;
        const float4* src = reinterpret_cast<const float4*>(qg + (int64_t)(live ? r >> 1 : 0) * kD + 384 + 64 * kb + 8 * c8);
        f[2 * t] = live ? src[0] : make_float4(0.f, 0.f, 0.f, 0.f);
        f[2 * t + 1] = live ? src[1] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int t = 0; t < kIt; ++t) {
      const int i = tid + t * kAtThreads;
      if (i < 128 * 16) {
        const int r = i >> 4, kb = (i >> 3) & 1, c8 = i & 7;
        uint32_t o[4];
        rope_q8(f[2 * t], f[2 * t + 1], p.rope_cs ? p.rope_cs + (int64_t)bt * 64 : nullptr, 48 + 8 * kb + c8);
        q_hilo_perm8(f[2 * t], f[2 * t + 1], r & 1, o);
        *reinterpret_cast<uint4*>(S.q2 + kb * kAtQBlkBytes + sw128_offset_h(r, 8 * c8)) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();                              // the indices and appended rows are ready

  if (warp == kAtWarpS) {
    // ------------------------------------------------------------ S2 issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(kFmtF16, kFmtF16, 128, kAtE);
      const uint32_t q2a = smem_u32(S.q2), kva = smem_u32(S.kv);
      for (int t = 0; t < nt; ++t) {
        const int bi = t & 1;
        if (!mbar_wait(kv_full + bi, (uint32_t)(t >> 1) & 1u, &g_at_error, kErrWaitTmaFull)) break;
        if (t >= 1 && !mbar_wait(s_free, (uint32_t)(t - 1) & 1u, &g_at_error, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t kvt = kva + (uint32_t)bi * kAtKVBytes;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t kb = ks >> 2, sub = ks & 3;
          const uint64_t bd = desc_k_sw128(kvt + kb * kAtKVBlk + sub * 32);
          if (kb < (uint32_t)kAtQTmemBlocks) {
            mma_f16_ts(tbase + kAtSCol, tbase + kb * 32 + sub * 8, bd, idesc_s, ks > 0 ? 1u : 0u);
          } else {
            const uint64_t ad = desc_k_sw128(q2a + (kb - kAtQTmemBlocks) * kAtQBlkBytes + sub * 32);
            mma_f16_ss(tbase + kAtSCol, ad, bd, idesc_s, 1u);
          }
        }
        mma_commit(s_full);
      }
      // every issued MMA has retired before the accumulators are released
      mma_commit(drain);
      mbar_wait(drain, 0u, &g_at_error, kErrWaitAccFull);
    }
  } else if (warp == kAtWarpPV) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_make_amn(kFmtF16, kFmtF16, 128, kAtH);
      const uint32_t kva = smem_u32(S.kv), pa = smem_u32(S.p);
      for (int i = 0; i < nt; ++i) {
        const int bi = i & 1;
        if (!mbar_wait(p_full + bi, (uint32_t)(i >> 1) & 1u, &g_at_error, kErrWaitAccFull)) break;
        tc_fence_after();
        const uint32_t kvt = kva + (uint32_t)bi * kAtKVBytes, pb = pa + (uint32_t)bi * 2 * kAtPBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int ks = 0; ks < kAtE / 16; ++ks) {
            // A = V^T: positions 128c.. (two 64-position blocks), entries 16ks..
            const uint64_t ad = desc_mn_sw128(kvt + (uint32_t)(2 * c) * kAtKVBlk + (uint32_t)ks * 2048, kAtKVBlk, 1024);
            // B = P^T hi, then lo: 64 head rows of 64 entries (128-byte swizzle), entries 16ks..
            const uint64_t bh = desc_k_sw128(pb + (uint32_t)ks * 32);
            const uint64_t bl = desc_k_sw128(pb + kAtPBytes + (uint32_t)ks * 32);
            mma_f16_ss(tbase + kAtOCol + 64u * c, ad, bh, idesc_o, (i > 0 || ks > 0) ? 1u : 0u);
            mma_f16_ss(tbase + kAtOCol + 64u * c, ad, bl, idesc_o, 1u);
          }
        }
        mma_commit(kv_free + bi);
        mma_commit(o_done);
      }
      mma_commit(drain + 1);
      mbar_wait(drain + 1, 0u, &g_at_error, kErrWaitAccFull);
    }
  } else if (is_deq) {
    // --------------------------------------------------- gather + dequantise
    if (!p.q2 && nt > 0) CSA_AT_FETCH(tile0);
    for (int i = 0; i < nt; ++i) {
      const int bi = i & 1;
      if (i >= 2 && !mbar_wait_warp(kv_free + bi, (uint32_t)((i >> 1) - 1) & 1u, kErrWaitSmemEmpty)) break;
      uint8_t* kt = S.kv + bi * kAtKVBytes;
      // this lane's staged codes (its own cp.async copies: no barrier needed)
      cp_async_wait_all();
      uint4 rr[8];
      {
        const uint8_t* rs = S.raw + 128 * (jd & 255);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          rr[k] = (k < 4 || kind == 2) ? *reinterpret_cast<const uint4*>(rs + 16 * (k ^ swz)) : make_uint4(0, 0, 0, 0);
      }
      // channels [128*q4, 128*q4 + 128) of entry e, one 16-byte chunk (8
      // positions) per group of 8 channels
      if (kind == 1) {
#pragma unroll
        for (int wq = 0; wq < 16; ++wq) {
          const uint4 r4 = rr[wq >> 2];
          const uint32_t w = (wq & 3) == 0 ? r4.x : (wq & 3) == 1 ? r4.y : (wq & 3) == 2 ? r4.z : r4.w;
          // block scale s (16 channels) as fp16 s * 2^7 (exact: s <= 448 < 2^9)
          const int sb = wq >> 1;
          uint32_t sc = ((sb < 4 ? rex.x : rex.y) >> (8 * (sb & 3))) & 0xFFu;
          sc |= sc << 16;
          const __half2 s2 = __hmul2(u2h(e4m3x2_bits_m8(sc)), u2h(kH2Exp15));
          // (E2M1 * 2^-14) * (s * 2^7) = E2M1 * s * 2^-7: at most 6
          // significant bits and >= 2^-17, so exact in fp16
          const uint32_t o0 = h2u(__hmul2(u2h(e2m1_pair_m14<0>(w)), s2));
          const uint32_t o1 = h2u(__hmul2(u2h(e2m1_pair_m14<1>(w)), s2));
          const uint32_t o2 = h2u(__hmul2(u2h(e2m1_pair_m14<2>(w)), s2));
          const uint32_t o3 = h2u(__hmul2(u2h(e2m1_pair_m14<3>(w)), s2));
          const int d = 128 * q4 + 8 * wq;
          *reinterpret_cast<uint4*>(kt + (uint32_t)(d >> 6) * kAtKVBlk + sw128_offset_h(e, d & 63)) =
              make_uint4(o0, o1, o2, o3);
        }
      } else if (kind == 2) {
#pragma unroll
        for (int g = 0; g < 16; ++g) {                // 8 code bytes = 8 channels
          const uint4 r4 = rr[g >> 1];
          const uint32_t w0 = (g & 1) ? r4.z : r4.x, w1 = (g & 1) ? r4.w : r4.y;   // channels 0-3, 4-7
          const int ex = (int)((rex.x >> (8 * (g >> 2))) & 0xFF);   // UE8M0: scale 2^(ex - 127)
          uint32_t o[4];
          if (ex >= 105 && ex <= 134) {
            // E4M3 * 2^-8 times the fp16 power of two 2^(ex - 119)
            const uint32_t f = (uint32_t)(ex - 104) << 10;
            const __half2 f2 = u2h(f | (f << 16));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              o[k] = h2u(__hmul2(u2h(e4m3x2_bits_m8(__byte_perm(w0, w1, k | (k << 4) | ((4 + k) << 8) | ((4 + k) << 12)))), f2));
          } else {
            // scales far from 1: fp32 product, rounded to fp16
            const float scf = exp2f((float)(ex - 127));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t two = ((w0 >> (8 * k)) & 0xFF) | (((w1 >> (8 * k)) & 0xFF) << 8);
              const float2 f = __half22float2(dec_e4m3x2(two));
              o[k] = h2u(__floats2half2_rn(f.x * scf, f.y * scf));
            }
          }
          const int d = 128 * q4 + 8 * g;
          *reinterpret_cast<uint4*>(kt + (uint32_t)(d >> 6) * kAtKVBlk + sw128_offset_h(e, d & 63)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int d = 128 * q4 + 8 * k;
          *reinterpret_cast<uint4*>(kt + (uint32_t)(d >> 6) * kAtKVBlk + sw128_offset_h(e, d & 63)) =
              make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(kv_full + bi);
      if (i + 1 < nt) CSA_AT_FETCH(tile0 + i + 1);
    }
    cp_async_wait_all();    // none in flight when the CTA leaves (also after an early break)
  } else {
    // ---------------------------------------------------------------- softmax
    const int qtr = warp;                      // TMEM lanes 32*qtr .. +31
    const int hp = 16 * qtr + (lane >> 1);     // head of this lane's Q2 row
    const int part = lane & 1;                 // row part (hi / lo) and entry half
    const uint32_t trow = tbase + ((uint32_t)(32 * qtr) << 16);
    const float sc_main = p.scale_log2 * 128.f, sc_win = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;      // l_run: this lane's entry half
    bool ok = true;
    // selected positions of entries `lane` and `lane + 32` of the next tile
    // (window entries: 0 when the row exists)
    int pos_a = -1, pos_b = -1;
    auto load_pos = [&](int tile) {
      const int ja = tile * kAtE + lane, jb = ja + 32;
      pos_a = ja < p.K ? idx_b[ja] : (ja < p.n_entries ? 0 : -1);
      pos_b = jb < p.K ? idx_b[jb] : (jb < p.n_entries ? 0 : -1);
    };
    if (nt > 0) load_pos(tile0);
    for (int i = 0; i < nt; ++i) {
      const int bi = i & 1;
      const uint32_t vm_a = __ballot_sync(0xffffffffu, pos_a >= 0);
      const uint32_t vm_b = __ballot_sync(0xffffffffu, pos_b >= 0);
      if (i + 1 < nt) load_pos(tile0 + i + 1);
      // a failed wait leaves `ok` false and skips the later waits, but every
      // warp still passes the group's named barriers once per tile
      ok = ok && mbar_wait_warp(s_full, (uint32_t)i & 1u, kErrWaitAccFull);
      tc_fence_after();
      // this lane takes entries [32*part, 32*part + 32) and adds the partner
      // row's logits for them; one 32-column load per half
      const uint32_t vmask = part ? vm_b : vm_a;
      const int jbase = (tile0 + i) * kAtE + 32 * part;
      const int n_main = p.K - jbase;          // entries below n_main are main (FP4) entries
      float x[32];
#pragma unroll
      for (int rnd = 0; rnd < 2; ++rnd) {
        uint32_t sv[32];
        tmem_ld32(trow + kAtSCol + 32 * rnd, sv);
        tmem_wait_ld();
        if (rnd == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
        const bool mine = rnd == part;          // columns 32rnd.. are this lane's entries
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float v = __uint_as_float(sv[k]);
          const float sum = v + __shfl_xor_sync(0xffffffffu, v, 1);
          if (mine) x[k] = sum;
        }
      }
      float mt = -INFINITY;
#pragma unroll
      for (int en = 0; en < 32; ++en) {
        const float v = ((vmask >> en) & 1u) ? x[en] * (en < n_main ? sc_main : sc_win) : -INFINITY;
        x[en] = v;
        mt = fmaxf(mt, v);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      bool need = false;
      float alpha = 1.f;
      if (mt > m_run + kAtRescale || (m_run == -INFINITY && mt > -INFINITY)) {
        alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - mt);
        m_run = mt;
        need = i > 0;
      }
      // rescale factors by tile parity: after this tile's reduction barrier a
      // warp may already write the next tile's factors while another still
      // reads these
      if (part == 0) S.alpha_s[64 * bi + hp] = alpha;
      float ls = 0.f;
#pragma unroll
      for (int en = 0; en < 32; ++en) {
        const float pe = (m_run == -INFINITY) ? 0.f : ex2_approx(x[en] - m_run);
        ls += pe;
        x[en] = en < n_main ? pe * 128.f : pe;
      }
      l_run = l_run * alpha + ls;
      // the P buffer is free once the PV two tiles back has retired
      if (i >= 2) ok = ok && mbar_wait_warp(kv_free + bi, (uint32_t)((i >> 1) - 1) & 1u, kErrWaitSmemEmpty);
      {
        // P as fp16 hi + lo parts (~22 bits): with fp16 P alone the weights'
        // rounding (2^-12) shows in channels whose entries are large but
        // whose weighted sum cancels
        uint8_t* pt = S.p + bi * 2 * kAtPBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t oh[4], ol[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a0 = x[8 * c + 2 * k], a1 = x[8 * c + 2 * k + 1];
            const __half2 hh = __floats2half2_rn(a0, a1);
            const float2 hf = __half22float2(hh);
            oh[k] = h2u(hh);
            ol[k] = h2u(__floats2half2_rn(a0 - hf.x, a1 - hf.y));
          }
          const uint32_t off = sw128_offset_h(hp, 32 * part + 8 * c);
          *reinterpret_cast<uint4*>(pt + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
          *reinterpret_cast<uint4*>(pt + kAtPBytes + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        }
      }
      // any head whose running max moved rescales the accumulated O^T columns
      // (after the previous tile's PV has retired)
      uint32_t any_need;
      asm volatile("{\n .reg .pred q, r;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred r, 1, 128, q;\n selp.u32 %0, 1, 0, r;\n}"
                   : "=r"(any_need) : "r"(need ? 1u : 0u) : "memory");
      if (any_need) {
        ok = ok && mbar_wait_warp(o_done, (uint32_t)(i - 1) & 1u, kErrWaitAccFull);
        tc_fence_after();
        // 16 heads at a time: their factors stay in registers across the 4 chunks
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          float al[16];
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) al[cc] = S.alpha_s[64 * bi + 16 * k + cc];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t ta = trow + kAtOCol + 64 * c + 16 * k;
            uint32_t o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) o[cc] = __float_as_uint(__uint_as_float(o[cc]) * al[cc]);
            tmem_st16(ta, o);
          }
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + bi);
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    const int h = hp;
    // ------------------------------------------------------------- output
    // per-head output scale (normalised, sink folded in) and lse, or partials
    if (part == 0) {
      float scl = 1.f;
      if (p.n_splits == 1) {
        float m0 = m_run, l0 = l_run;
        if (p.sink && h < H) {
          const float s0 = p.sink[h] * kAtLog2e;
          const float n0 = fmaxf(m0, s0);
          l0 = (l0 > 0.f ? l0 * exp2f(m0 - n0) : 0.f) + (s0 == -INFINITY ? 0.f : exp2f(s0 - n0));
          scl = (m0 == -INFINITY || l0 <= 0.f) ? 0.f : exp2f(m0 - n0) / l0;
          m0 = n0;
        } else {
          scl = l0 > 0.f ? 1.f / l0 : 0.f;
        }
        if (p.lse && h < H) p.lse[(int64_t)bt * H + h] = l0 > 0.f ? (m0 + log2f(l0)) * kAtLn2 : -INFINITY;
      } else if (h < H) {
        *reinterpret_cast<float2*>(p.part_ml + (((int64_t)bt * p.n_splits + split) * H + h) * 2) =
            make_float2(m_run, l_run);
      }
      S.scl[h] = scl;
    }
    named_bar(1, 128);
    // every thread waits for the last PV itself (no wait is skipped on an
    // error), on the PV issuer's single-phase drain barrier: o_done completes
    // once per tile and a parity wait on it cannot tell whether the PV before
    // the last one has retired (a last tile without a rescale never waited
    // for it), so it could return while that PV still accumulates.
    if (ok && nt > 0) ok = mbar_wait_warp(drain + 1, 0u, kErrWaitAccFull);
    tc_fence_after();
    if (p.n_splits == 1) {
      for (int c = 0; c < 4; ++c) {
        // O^T row (position) 128c + 32qtr + lane holds this latent channel
        const int dp = 128 * c + 32 * qtr + lane;
        const int d = (dp & ~7) | perm8(dp & 7);
        // 64 heads of channel d: one 64-column load
        uint32_t o[64];
        if (nt > 0 && ok) {
          tmem_ld64(trow + kAtOCol + 64 * c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 64; ++k) o[k] = 0u;
        }
#pragma unroll
        for (int hd = 0; hd < kAtH; ++hd) o[hd] = __float_as_uint(__uint_as_float(o[hd]) * S.scl[hd]);
        if (p.rope_cs && c == 3 && qtr >= 2) {
          // channels 448..511: channel d ^ 1 of the rotated pair sits in lane ^ 2
          const float2 k = *reinterpret_cast<const float2*>(p.rope_cs + (int64_t)bt * 64 + ((d - kRopeStart) & ~1));
#pragma unroll
          for (int hd = 0; hd < kAtH; ++hd) {
            const float v = __uint_as_float(o[hd]);
            const float pv = __shfl_xor_sync(0xffffffffu, v, 2);
            o[hd] = __float_as_uint((d & 1) ? v * k.x - pv * k.y : v * k.x + pv * k.y);
          }
        }
        const int64_t base = (int64_t)bt * H * kD + d;
#pragma unroll
        for (int hd = 0; hd < kAtH; ++hd)
          if (hd < H) store_out1(p.out, p.out_bf16, base + (int64_t)hd * kD, __uint_as_float(o[hd]));
      }
    } else if (!ok || nt == 0) {
      *S.o_bad = 1;
    }
  }
  if (p.n_splits > 1) {
    // ------------------------------------------------------ partial O^T
    // the softmax warps have seen the last PV retire; warps w and w + 4 share
    // TMEM lane quarter w & 3 and write chunks {0, 1} and {2, 3} as
    // [head][channel] rows straight from their TMEM rows: per head a warp
    // stores 32 neighbouring channels (128 contiguous bytes).  Staging the
    // rows in shared memory for one bulk copy was slower: the copy moved the
    // 128 KB no faster than these stores, after the staging.
    __syncthreads();
    if (warp < 8) {
      const int qq = warp & 3, cb = 2 * (warp >> 2);
      const bool valid = *S.o_bad == 0;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = cb + cc;
        const int dp = 128 * c + 32 * qq + lane;
        const int d = (dp & ~7) | perm8(dp & 7);
        uint32_t o[64];
        if (valid) {
          tmem_ld64(tbase + ((uint32_t)(32 * qq) << 16) + kAtOCol + 64 * c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 64; ++k) o[k] = 0u;
        }
        float* po = p.part_o + ((int64_t)bt * p.n_splits + split) * H * kD + d;
#pragma unroll
        for (int hd = 0; hd < kAtH; ++hd)
          if (hd < H) po[(int64_t)hd * kD] = __uint_as_float(o[hd]);
      }
    }
  }
#undef CSA_AT_FETCH
  tc_fence_before();
  __syncthreads();
  if (warp == kAtWarpS) {
    tc_fence_after();
    tmem_dealloc(tbase, kAtTmemCols);
  }
}

size_t attn_tc_smem_bytes() { return kAtSmemBytes; }

cudaError_t launch_attn_tc(const AttnTcParams& p, cudaStream_t stream) {
  static SmemAttrOnce attr;
  const cudaError_t ea = attr.set(sparse_attn_tc_kernel, kAtSmemBytes);
  if (ea != cudaSuccess) return ea;
  dim3 grid(p.n_splits, p.B * p.n_q);
  ProfScope ps(stream, "sparse_attn_tc");
  launch_k(sparse_attn_tc_kernel, grid, dim3(kAtThreads), kAtSmemBytes, stream, p);
  note_launches(1);
  return cudaGetLastError();
}

int read_at_error(bool clear) {
  int v = 0;
  cudaMemcpyFromSymbol(&v, g_at_error, sizeof(int));
  if (clear && v) {
    int z = 0;
    cudaMemcpyToSymbol(g_at_error, &z, sizeof(int));
  }
  return v;
}

}  // namespace csa
