// Sparse MLA attention on the 5th-generation tensor cores (tcgen05), for 64
// query heads (the shape of the step's attention layers).
//
// Same function as sparse_attn_mma_kernel (MLA over the Top-K selected FP4
// entries plus the FP8 window, K = V = the 512-wide latent; Model techniques
// map - DeepSeek-V4.1-Flash, "Multi-head latent attention", "Indexer-selected
// sparse attention", "Sliding-window attention" and "Learnable attention
// sink" rows).  Per 32-entry tile of one token:
//   S2 = Q2 K^T   tcgen05.mma kind::f16, M = 128 rows of Q2: row 2h is the
//                 fp16 hi part of head h's query, row 2h+1 the lo part
//                 fp16(q - hi); N = 32 entries, K = 512; fp32 in TMEM.  The
//                 softmax adds the two rows of a head (neighbouring lanes of
//                 one warp), which carries ~22 bits of q against the exactly
//                 dequantised fp16 entries.
//   O^T += V^T P^T  tcgen05.mma kind::f16, M = 128 latent channels (4
//                 chunks), N = 64 heads, K = 32 entries, fp32 in TMEM.  The
//                 same shared-memory tile of dequantised entries is the
//                 K-major B operand of S2 and the MN-major A operand here.
// Warp roles: warps 0-3 softmax / output (one TMEM lane quarter each; the
// two lanes of a head split the tile's entries), warps 4-7 gather +
// dequantise (8 threads per 8 entries and 128 channels; the next tile's raw
// bytes are loaded into registers while the current one is decoded), warp 8
// issues the S2 MMAs, warp 9 the PV MMAs.  The entry tile, P and S are
// double buffered, so tile i+1 is dequantised and its S2 computed while the
// softmax and PV of tile i run.  Online softmax in the exp2 domain with lazy
// rescaling: the running max only moves when a tile's max exceeds it by more
// than 8, and only then are the O^T accumulators rescaled in TMEM.
//
// Main (FP4) entries are staged as E2M1 * s * 2^-7 (exact in fp16, one
// multiply per channel pair); their logits are scaled by 2^7 and their
// probabilities by 2^7 in P, which leaves S and O unchanged.  Window entries
// are staged unscaled.  All waits are bounded (sm100.cuh).
#include "sm100.cuh"
#include "attn_tc.cuh"

namespace csa {


constexpr int kAtH = 64;                  // heads
constexpr int kAtE = 32;                  // entries per tile
constexpr int kAtThreads = 320;           // 10 warps
constexpr int kAtQBytes = 128 * 512 * 2;  // Q2: 128 rows x 512 fp16
constexpr int kAtKVBytes = kAtE * 512 * 2;        // one entry tile (8 blocks of 64 channels)
constexpr int kAtKVBlk = kAtE * 128;              // bytes of one 64-channel block
constexpr int kAtPBytes = kAtH * kAtE * 2;        // one P^T tile: 64 head rows x 64 B
constexpr int kAtXSBytes = kAtE * kAtH * 4;
constexpr size_t kAtSmemBytes = 1024 + kAtQBytes + 2 * kAtKVBytes + 2 * kAtPBytes + kAtXSBytes + 1024;
constexpr uint32_t kAtTmemCols = 512;     // S buffers: cols 0..31, 32..63; O^T chunk c: cols 64 + 64c
constexpr uint32_t kAtOCol = 64;
constexpr float kAtLog2e = 1.4426950408889634f;
constexpr float kAtLn2 = 0.6931471805599453f;
constexpr float kAtRescale = 8.0f;        // lazy-rescale threshold (exp2 units)

static __device__ int g_at_error;

struct AtSmem {
  uint8_t* q2;
  uint8_t* kv;      // 2 buffers
  uint8_t* p;       // 2 buffers
  float* xs;        // [entry][head] lo-part logits
  float* scl;       // [64] per-head output scale
  float* alpha_s;   // [64]
  uint64_t* bars;
  uint32_t* tmem_base;
};

CSA_DEV AtSmem carve_at(uint8_t* raw) {
  AtSmem s;
  uintptr_t base = (reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  s.q2 = p; p += kAtQBytes;
  s.kv = p; p += 2 * kAtKVBytes;
  s.p = p; p += 2 * kAtPBytes;
  s.xs = reinterpret_cast<float*>(p); p += kAtXSBytes;
  s.scl = reinterpret_cast<float*>(p); p += 64 * 4;
  s.alpha_s = reinterpret_cast<float*>(p); p += 64 * 4;
  s.bars = reinterpret_cast<uint64_t*>(p); p += 16 * 8;
  s.tmem_base = reinterpret_cast<uint32_t*>(p);
  return s;
}

CSA_DEV uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
CSA_DEV __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Integer-pipe decoders (the conversion pipe is the scarce one here).
// A 4-bit E2M1 code n placed at bits 0-3 (and 16-19) becomes the fp16 value
// E2M1(n) * 2^-14 by moving its magnitude bits to fp16 bits 9-11 and its sign
// to bit 15: E2M1's exponent field lines up with the low fp16 exponent bits
// and its subnormal (0.5) with the fp16 subnormal 2^-15.
CSA_DEV uint32_t e2m1x2_bits_m14(uint32_t t) {
  return ((t << 9) & 0x0E000E00u) | ((t << 12) & 0x80008000u);
}
// An 8-bit E4M3 code c at bits 0-7 (and 16-23) becomes the fp16 value
// E4M3(c) * 2^-8 the same way (exponent and mantissa shifted by 7, sign to
// bit 15); E4M3 subnormals land on fp16 subnormals, so every code is exact.
CSA_DEV uint32_t e4m3x2_bits_m8(uint32_t t) {
  return ((t << 7) & 0x3F803F80u) | ((t << 8) & 0x80008000u);
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
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  AtSmem S = carve_at(smem_raw);
  uint64_t* kv_full = S.bars + 0;    // [2] dequant -> MMA (4 warp arrivals)
  uint64_t* kv_free = S.bars + 2;    // [2] PV done: entry tile and P buffer reusable
  uint64_t* s_full = S.bars + 4;     // [2] S2 in TMEM
  uint64_t* s_free = S.bars + 6;     // [2] S2 read by the softmax (4 warp arrivals)
  uint64_t* p_full = S.bars + 8;     // [2] P written, O^T rescaled (4 warp arrivals)
  uint64_t* o_done = S.bars + 10;    // one phase per PV
  uint64_t* drain = S.bars + 11;     // [2] all MMAs of an issuer retired (teardown)
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
      mbar_init(kv_full + k, 4);
      mbar_init(kv_free + k, 1);
      mbar_init(s_full + k, 1);
      mbar_init(s_free + k, 4);
      mbar_init(p_full + k, 4);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    mbar_init(drain + 1, 1);
    fence_mbar_init();
  }
  // gather role: 8 consecutive lanes take 8 different entries, so each
  // quarter-warp phase of a 16-byte shared store covers all 32 banks
  const int jd = tid - 128;
  const int e = 8 * (jd >> 5) + (jd & 7), q4 = (jd >> 3) & 3;   // entry, quarter (128 channels)
  const int32_t* idx_b = p.idx + (int64_t)bt * p.K;
  const uint8_t* kvb = p.kv + (int64_t)b * p.kv_batch_stride;
  const uint8_t* wb = p.win ? p.win + (int64_t)b * p.win_batch_stride : nullptr;
  uint4 rr[8];
  uint2 rex = make_uint2(0, 0);
  int kind = 0;   // 0 invalid, 1 FP4 main entry, 2 FP8 window entry
#define CSA_AT_FETCH(tile)                                                                     \
  do {                                                                                         \
    const int jj = (tile) * kAtE + e;                                                          \
    kind = 0;                                                                                  \
    if (jj < p.K) {                                                                            \
      const int pos = idx_b[jj];                                                               \
      if (pos >= 0) {                                                                          \
        const uint8_t* row = kvb + (int64_t)pos * p.kv_row_stride;                             \
        _Pragma("unroll") for (int k = 0; k < 4; ++k) rr[k] = ld_nc_v4(row + 64 * q4 + 16 * k); \
        rex = *reinterpret_cast<const uint2*>(row + 256 + 8 * q4);                             \
        kind = 1;                                                                              \
      }                                                                                        \
    } else if (jj < p.n_entries) {                                                             \
      const uint8_t* row = wb + (int64_t)(tq + jj - p.K) * p.win_row_stride;                   \
      _Pragma("unroll") for (int k = 0; k < 8; ++k) rr[k] = ld_nc_v4(row + 128 * q4 + 16 * k); \
      rex.x = *reinterpret_cast<const uint32_t*>(row + 512 + 4 * q4);                          \
      kind = 2;                                                                                \
    }                                                                                          \
  } while (0)
  // the first tile's entries are in flight while q is staged
  if (warp >= 4 && warp < 8 && nt > 0) CSA_AT_FETCH(tile0);
  // Q2 rows (2h, 2h+1) = (hi, lo) of head h, fp16, K-major 128-byte swizzle,
  // 8 blocks of 64 channels
  {
    const float* qg = p.q + (int64_t)bt * kAtH * kD;
#pragma unroll 2
    for (int i = tid; i < kAtH * (kD / 8); i += kAtThreads) {
      const int h = i / (kD / 8), c8 = i % (kD / 8);        // 8 channels at 8*c8
      const float4 a = reinterpret_cast<const float4*>(qg + (int64_t)h * kD + 8 * c8)[0];
      const float4 c = reinterpret_cast<const float4*>(qg + (int64_t)h * kD + 8 * c8)[1];
      const float f[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hh = __floats2half2_rn(f[2 * k], f[2 * k + 1]);
        const float2 hf = __half22float2(hh);
        hi[k] = h2u(hh);
        lo[k] = h2u(__floats2half2_rn(f[2 * k] - hf.x, f[2 * k + 1] - hf.y));
      }
      const int d = 8 * c8;
      const uint32_t blk = (uint32_t)(d >> 6) * (128 * 128);
      *reinterpret_cast<uint4*>(S.q2 + blk + sw128_offset_h(2 * h, d & 63)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(S.q2 + blk + sw128_offset_h(2 * h + 1, d & 63)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  fence_proxy_async_smem();
  if (warp == 8) tmem_alloc(S.tmem_base, kAtTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *S.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ S2 issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(kFmtF16, kFmtF16, 128, kAtE);
      const uint32_t q2a = smem_u32(S.q2), kva = smem_u32(S.kv);
      for (int t = 0; t < nt; ++t) {
        const int bi = t & 1, ui = t >> 1;
        if (!mbar_wait(kv_full + bi, (uint32_t)ui & 1u, &g_at_error, kErrWaitTmaFull)) break;
        if (t >= 2 && !mbar_wait(s_free + bi, (uint32_t)(ui - 1) & 1u, &g_at_error, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t kvb = kva + (uint32_t)bi * kAtKVBytes;
#pragma unroll 4
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t kb = ks >> 2, sub = ks & 3;
          const uint64_t ad = desc_k_sw128(q2a + kb * (128 * 128) + sub * 32);
          const uint64_t bd = desc_k_sw128(kvb + kb * kAtKVBlk + sub * 32);
          mma_f16_ss(tbase + 32u * bi, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full + bi);
      }
      // every issued MMA has retired before the accumulators are released
      mma_commit(drain);
      mbar_wait(drain, 0u, &g_at_error, kErrWaitAccFull);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_make_amn(kFmtF16, kFmtF16, 128, kAtH);
      const uint32_t kva = smem_u32(S.kv), pa = smem_u32(S.p);
      for (int i = 0; i < nt; ++i) {
        const int bi = i & 1;
        if (!mbar_wait(p_full + bi, (uint32_t)(i >> 1) & 1u, &g_at_error, kErrWaitAccFull)) break;
        tc_fence_after();
        const uint32_t kvb = kva + (uint32_t)bi * kAtKVBytes, pb = pa + (uint32_t)bi * kAtPBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int ks = 0; ks < kAtE / 16; ++ks) {
            // A = V^T: channels 128c.. (two 64-channel blocks), entries 16ks..
            const uint64_t ad = desc_mn_sw128(kvb + (uint32_t)(2 * c) * kAtKVBlk + (uint32_t)ks * 2048, kAtKVBlk, 1024);
            // B = P^T: 64 head rows of 32 entries (64-byte swizzle), entries 16ks..
            const uint64_t bd = desc_k_sw64(pb + (uint32_t)ks * 32);
            mma_f16_ss(tbase + kAtOCol + 64u * c, ad, bd, idesc_o, (i > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(kv_free + bi);
        mma_commit(o_done);
      }
      mma_commit(drain + 1);
      mbar_wait(drain + 1, 0u, &g_at_error, kErrWaitAccFull);
    }
  } else if (warp >= 4) {
    // --------------------------------------------------- gather + dequantise
    for (int i = 0; i < nt; ++i) {
      const int bi = i & 1;
      if (i >= 2 && !mbar_wait_warp(kv_free + bi, (uint32_t)((i >> 1) - 1) & 1u, kErrWaitSmemEmpty)) break;
      uint8_t* kt = S.kv + bi * kAtKVBytes;
      // channels [128*q4, 128*q4 + 128) of entry e -> fp16 at (e, d)
      if (kind == 1) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {                 // 16 code bytes = 32 channels = 2 scale blocks
          const uint32_t cw[4] = {rr[k].x, rr[k].y, rr[k].z, rr[k].w};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // block scale s as fp16 s * 2^7 (exact: s <= 448 < 2^9)
            const int sb = 2 * k + half;
            uint32_t sc = ((sb < 4 ? rex.x : rex.y) >> (8 * (sb & 3))) & 0xFFu;
            sc |= sc << 16;
            const __half2 s2 = __hmul2(u2h(e4m3x2_bits_m8(sc)), u2h(kH2Exp15));
#pragma unroll
            for (int wi = 0; wi < 2; ++wi) {           // one word = 8 channels
              const uint32_t w = cw[2 * half + wi];
              const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
              uint32_t o[4];
#pragma unroll
              for (int bb = 0; bb < 4; ++bb) {
                // channels 2bb, 2bb+1 of the word: low nibble -> low half
                const uint32_t t = __byte_perm(lo, hi, bb | (bb << 4) | ((4 + bb) << 8) | ((4 + bb) << 12));
                // (E2M1 * 2^-14) * (s * 2^7) = E2M1 * s * 2^-7: at most 6
                // significant bits and >= 2^-17, so exact in fp16
                o[bb] = h2u(__hmul2(u2h(e2m1x2_bits_m14(t)), s2));
              }
              const int d = 128 * q4 + 32 * k + 16 * half + 8 * wi;
              *reinterpret_cast<uint4*>(kt + (uint32_t)(d >> 6) * kAtKVBlk + sw128_offset_h(e, d & 63)) =
                  make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      } else if (kind == 2) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {                 // 16 code bytes = 16 channels
          const int ex = (int)((rex.x >> (8 * (k >> 1))) & 0xFF);   // UE8M0: scale 2^(ex - 127)
          const uint32_t cw[4] = {rr[k].x, rr[k].y, rr[k].z, rr[k].w};
          uint32_t o[8];
          if (ex >= 105 && ex <= 134) {
            // E4M3 * 2^-8 times the fp16 power of two 2^(ex - 119)
            const uint32_t f = (uint32_t)(ex - 104) << 10;
            const __half2 f2 = u2h(f | (f << 16));
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              o[2 * wi] = h2u(__hmul2(u2h(e4m3x2_bits_m8(__byte_perm(cw[wi], 0u, 0x4140))), f2));
              o[2 * wi + 1] = h2u(__hmul2(u2h(e4m3x2_bits_m8(__byte_perm(cw[wi], 0u, 0x4342))), f2));
            }
          } else {
            // scales far from 1: fp32 product, rounded to fp16
            const float scf = exp2f((float)(ex - 127));
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
              const uint32_t two = (cw[bb >> 1] >> (16 * (bb & 1))) & 0xFFFF;
              const float2 f = __half22float2(dec_e4m3x2(two));
              o[bb] = h2u(__floats2half2_rn(f.x * scf, f.y * scf));
            }
          }
#pragma unroll
          for (int half8 = 0; half8 < 2; ++half8) {
            const int d = 128 * q4 + 16 * k + 8 * half8;
            *reinterpret_cast<uint4*>(kt + (uint32_t)(d >> 6) * kAtKVBlk + sw128_offset_h(e, d & 63)) =
                make_uint4(o[4 * half8], o[4 * half8 + 1], o[4 * half8 + 2], o[4 * half8 + 3]);
          }
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
#undef CSA_AT_FETCH
  } else {
    // ---------------------------------------------------------------- softmax
    const int qtr = warp;                      // TMEM lanes 32*qtr .. +31
    const int hp = 16 * qtr + (lane >> 1);     // head of this lane's Q2 row
    const int part = lane & 1;                 // row part (hi / lo) and entry half
    const uint32_t trow = tbase + ((uint32_t)(32 * qtr) << 16);
    const float sc_main = p.scale_log2 * 128.f, sc_win = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;      // l_run: this lane's entry half
    bool ok = true;
    // selected position of entry `lane` of the next tile (window entries: row exists)
    int pos_next = 0;
    if (nt > 0) {
      const int jj = tile0 * kAtE + lane;
      pos_next = jj < p.K ? idx_b[jj] : (jj < p.n_entries ? 0 : -1);
    }
    for (int i = 0; i < nt; ++i) {
      const int bi = i & 1;
      const uint32_t vmask = __ballot_sync(0xffffffffu, pos_next >= 0);
      if (i + 1 < nt) {
        const int jj = (tile0 + i + 1) * kAtE + lane;
        pos_next = jj < p.K ? idx_b[jj] : (jj < p.n_entries ? 0 : -1);
      }
      // a failed wait leaves `ok` false and skips the later waits, but every
      // warp still passes the group's named barriers once per tile
      ok = ok && mbar_wait_warp(s_full + bi, (uint32_t)(i >> 1) & 1u, kErrWaitAccFull);
      tc_fence_after();
      float sv[kAtE];
#pragma unroll
      for (int k = 0; k < kAtE / 16; ++k) tmem_ld16f(trow + 32u * bi + 16 * k, sv + 16 * k);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + bi);
      // this lane takes entries [16*part, 16*part + 16): add the partner row's part
      const int jbase = (tile0 + i) * kAtE + 16 * part;
      const int n_main = p.K - jbase;          // entries below n_main are main (FP4) entries
      float x[16];
      float mt = -INFINITY;
#pragma unroll
      for (int en = 0; en < 16; ++en) {
        const float send = part ? sv[en] : sv[16 + en];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
        const float sum = (part ? sv[16 + en] : sv[en]) + recv;
        const float v = ((vmask >> (16 * part + en)) & 1u) ? sum * (en < n_main ? sc_main : sc_win) : -INFINITY;
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
      if (part == 0) S.alpha_s[hp] = alpha;
      float ls = 0.f;
#pragma unroll
      for (int en = 0; en < 16; ++en) {
        const float pe = (m_run == -INFINITY) ? 0.f : ex2_approx(x[en] - m_run);
        ls += pe;
        x[en] = en < n_main ? pe * 128.f : pe;
      }
      l_run = l_run * alpha + ls;
      // the P buffer is free once the PV two tiles back has retired
      if (i >= 2) ok = ok && mbar_wait_warp(kv_free + bi, (uint32_t)((i >> 1) - 1) & 1u, kErrWaitSmemEmpty);
      {
        uint8_t* pt = S.p + bi * kAtPBytes;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) o[k] = h2u(__floats2half2_rn(x[8 * c + 2 * k], x[8 * c + 2 * k + 1]));
          *reinterpret_cast<uint4*>(pt + sw64_offset(hp, 32 * part + 16 * c)) = make_uint4(o[0], o[1], o[2], o[3]);
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
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t ta = trow + kAtOCol + 64 * c + 16 * k;
            uint32_t o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) o[cc] = __float_as_uint(__uint_as_float(o[cc]) * S.alpha_s[16 * k + cc]);
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
    const bool is_hi = part == 0;
    // ------------------------------------------------------------- output
    // per-head output scale (normalised, sink folded in) and lse, or partials
    if (is_hi) {
      float scl = 1.f;
      if (p.n_splits == 1) {
        float m0 = m_run, l0 = l_run;
        if (p.sink) {
          const float s0 = p.sink[h] * kAtLog2e;
          const float n0 = fmaxf(m0, s0);
          l0 = (l0 > 0.f ? l0 * exp2f(m0 - n0) : 0.f) + (s0 == -INFINITY ? 0.f : exp2f(s0 - n0));
          scl = (m0 == -INFINITY || l0 <= 0.f) ? 0.f : exp2f(m0 - n0) / l0;
          m0 = n0;
        } else {
          scl = l0 > 0.f ? 1.f / l0 : 0.f;
        }
        if (p.lse) p.lse[(int64_t)bt * kAtH + h] = l0 > 0.f ? (m0 + log2f(l0)) * kAtLn2 : -INFINITY;
      } else {
        *reinterpret_cast<float2*>(p.part_ml + (((int64_t)bt * p.n_splits + split) * kAtH + h) * 2) =
            make_float2(m_run, l_run);
      }
      S.scl[h] = scl;
    }
    named_bar(1, 128);
    // every thread waits for the last PV itself (no wait is skipped on an error)
    if (ok && nt > 0) ok = mbar_wait_warp(o_done, ((uint32_t)(nt - 1) & 1u), kErrWaitAccFull);
    tc_fence_after();
    for (int c = 0; c < 4; ++c) {
      const int d = 128 * c + 32 * qtr + lane;
      // 64 heads of channel d: four loads in flight, one wait
      uint32_t o[64];
      if (nt > 0 && ok) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t (&ok16)[16] = *reinterpret_cast<uint32_t(*)[16]>(o + 16 * k);
          tmem_ld16(tbase + ((uint32_t)(32 * qtr) << 16) + kAtOCol + 64 * c + 16 * k, ok16);
        }
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) o[k] = 0u;
      }
      if (p.n_splits == 1) {
        float* dst = p.out + (int64_t)bt * kAtH * kD + d;
#pragma unroll
        for (int hd = 0; hd < kAtH; ++hd) dst[(int64_t)hd * kD] = __uint_as_float(o[hd]) * S.scl[hd];
      } else {
        float* dst = p.part_o + ((int64_t)bt * p.n_splits + split) * kAtH * kD + d;
#pragma unroll
        for (int hd = 0; hd < kAtH; ++hd) dst[(int64_t)hd * kD] = __uint_as_float(o[hd]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, kAtTmemCols);
  }
}

size_t attn_tc_smem_bytes() { return kAtSmemBytes; }

cudaError_t launch_attn_tc(const AttnTcParams& p, cudaStream_t stream) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(sparse_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAtSmemBytes);
    attr = true;
  }
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
